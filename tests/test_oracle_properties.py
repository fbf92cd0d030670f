"""Property-based pins of the oracle (hypothesis): for random shapes, degrees
and packings the sharded layers equal the unsharded ones, the slices partition
the weight, and packed slices are permutations of its rows / columns.  These
hold exactly on small-integer inputs, where float64 arithmetic is exact."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as o


def _ints(rng, shape):
    return rng.integers(-3, 4, size=shape).astype(np.float64)


@settings(max_examples=60, deadline=None)
@given(T=st.sampled_from([1, 2, 3, 4, 6]), m=st.integers(1, 6), k=st.integers(1, 4), n=st.integers(1, 4),
       seed=st.integers(0, 2**31 - 1))
def test_colwise_rowwise_pair_equals_unsharded(T, m, k, n, seed):
    rng = np.random.default_rng(seed)
    D, F = k * T, n * T
    X, W_up, W_down = _ints(rng, (m, D)), _ints(rng, (F, D)), _ints(rng, (D, F))
    b_up, b_down = _ints(rng, (F,)), _ints(rng, (D,))
    ident = lambda x: x  # noqa: E731  (exact: no transcendental)
    full = o.mlp_unsharded(X, W_up, b_up, W_down, b_down, act=ident)
    tp = o.mlp_sharded_summed(X, W_up, b_up, W_down, b_down, T, act=ident)
    assert np.array_equal(full, tp)


@settings(max_examples=60, deadline=None)
@given(T=st.sampled_from([1, 2, 4]), blocks=st.lists(st.integers(1, 4), min_size=1, max_size=5),
       unit=st.integers(1, 3), cols=st.integers(1, 5), seed=st.integers(0, 2**31 - 1))
def test_packed_slices_partition_the_weight(T, blocks, unit, cols, seed):
    rng = np.random.default_rng(seed)
    sizes = [b * unit * T for b in blocks]           # every block divisible by T
    P = sum(sizes)
    W = np.arange(P * cols).reshape(P, cols)
    rows = np.concatenate([o.slice_packed_colwise(W, sizes, T, r) for r in range(T)])
    assert sorted(rows[:, 0].tolist()) == sorted(W[:, 0].tolist())   # each row exactly once
    Wt = W.T.copy()
    cols_ = np.concatenate([o.slice_packed_rowwise(Wt, sizes, T, r) for r in range(T)], axis=1)
    assert sorted(cols_[0].tolist()) == sorted(Wt[0].tolist())
    # shard r holds, for every block in order, that block's r-th contiguous part
    for r in range(T):
        part = o.slice_packed_colwise(W, sizes, T, r)
        start = off = 0
        for s in sizes:
            q = s // T
            assert np.array_equal(part[off:off + q], W[start + r * q:start + (r + 1) * q])
            start += s
            off += q


@settings(max_examples=40, deadline=None)
@given(T=st.sampled_from([1, 2, 3, 4]), m=st.integers(1, 5), k=st.integers(1, 4), n=st.integers(1, 5),
       seed=st.integers(0, 2**31 - 1))
def test_rowwise_split_input_equals_full_projection(T, m, k, n, seed):
    rng = np.random.default_rng(seed)
    X, W, b = _ints(rng, (m, k * T)), _ints(rng, (n, k * T)), _ints(rng, (n,))
    assert np.array_equal(o.rowwise_split_input(X, W, b, T), X @ W.T + b)


@settings(max_examples=25, deadline=None)
@given(T=st.sampled_from([1, 2]), mi=st.integers(1, 5), mt=st.integers(0, 4), seed=st.integers(0, 2**31 - 1))
def test_joint_sharded_equals_unsharded(T, mi, mt, seed):
    rng = np.random.default_rng(seed)
    D, heads = 256, 2
    w = lambda *s: rng.standard_normal(s) / np.sqrt(s[-1])  # noqa: E731
    Xi, Xt = rng.standard_normal((mi, D)), rng.standard_normal((mt, D))
    Wqi, Wqt, Woi, Wot = w(3 * D, D), w(3 * D, D), w(D, D), w(D, D)
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt, Wqi, Wqt, Woi, Wot, heads)
    Si, St = o.joint_attn_sharded_summed(Xi, Xt, Wqi, Wqt, Woi, Wot, heads, T)
    assert np.allclose(Yi, Si, rtol=1e-12, atol=1e-12) and np.allclose(Yt, St, rtol=1e-12, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(T=st.sampled_from([1, 2, 3, 4]), m=st.integers(1, 5), k=st.integers(1, 3), n=st.integers(1, 3),
       seed=st.integers(0, 2**31 - 1))
def test_colwise_shards_and_rowwise_partials_compose_the_layer(T, m, k, n, seed):
    # The two halves of the pair one at a time: each colwise shard is a column
    # block of the unsharded hidden layer, and the rowwise partials of those
    # blocks plus the bias once sum to the unsharded output (exact on integers).
    rng = np.random.default_rng(seed)
    D, F = k * T, n * T
    X, W_up, W_down = _ints(rng, (m, D)), _ints(rng, (F, D)), _ints(rng, (D, F))
    b_up, b_down = _ints(rng, (F,)), _ints(rng, (D,))
    ident = lambda x: x  # noqa: E731
    H_full = X @ W_up.T + b_up
    parts = []
    for r in range(T):
        H_r = o.mlp_colwise_shard(X, W_up, b_up, T, r, act=ident)
        assert np.array_equal(H_r, H_full[:, r * n:(r + 1) * n])
        parts.append(o.mlp_rowwise_partial(H_r, W_down, T, r))
    assert np.array_equal(sum(parts) + b_down, o.mlp_unsharded(X, W_up, b_up, W_down, b_down, act=ident))


@settings(max_examples=15, deadline=None)
@given(T=st.sampled_from([1, 2, 4]), m=st.integers(1, 6), seed=st.integers(0, 2**31 - 1))
def test_attention_shard_outputs_partition_the_heads(T, m, seed):
    # Head splitting is an exact partition: shard r's attention output is the
    # column block of its heads in the unsharded per-head output, each head
    # computed on its own (the attention of a head reads only that head's
    # Q, K and V columns).
    heads, dh = 4, 128
    D = heads * dh
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((m, D)) * 0.05
    W_qkv = rng.standard_normal((3 * D, D)) * 0.05
    qkv = X @ W_qkv.T
    full = np.concatenate([o.sdpa(qkv[:, h * dh:(h + 1) * dh], qkv[:, D + h * dh:D + (h + 1) * dh],
                                  qkv[:, 2 * D + h * dh:2 * D + (h + 1) * dh]) for h in range(heads)], axis=1)
    Hs = heads // T
    for r in range(T):
        O_r = o.attn_shard_output(X, W_qkv, heads, T, r)
        np.testing.assert_allclose(O_r, full[:, r * Hs * dh:(r + 1) * Hs * dh], rtol=1e-12, atol=1e-12)
