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
