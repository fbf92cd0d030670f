"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped bias, a bias
added per shard, a transposed weight, a wrong slice or head index, Q/K/V in the
wrong order, a wrong softmax scale, a wrong GELU constant) fails at least one of
them.  ``test_pins_have_teeth`` plants such slips in the oracle, on the CPU, and
checks that a pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as o
import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "slices.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# Slicing: hand-derived fixture + partition invariants.
# ---------------------------------------------------------------------------

def test_slices_match_hand_fixture():
    g = json.load(open(GOLDEN))
    W = np.arange(24).reshape(g["W_shape"])
    T = g["tp_degree"]
    for r in range(T):
        assert np.array_equal(o.slice_colwise(W, T, r), np.array(g["colwise"][str(r)]))
        assert np.array_equal(o.slice_rowwise(W, T, r), np.array(g["rowwise"][str(r)]))
    pc = g["packed_colwise"]
    Wp = np.arange(pc["rows"])[:, None] * np.ones((1, 3), dtype=np.int64)
    for r in range(T):
        got = o.slice_packed_colwise(Wp, pc["blocks"], T, r)[:, 0]
        assert list(got) == pc[str(r)]
    q = g["qkv_heads"]
    Wq = np.arange(3 * q["D"])[:, None] * np.ones((1, q["D"]), dtype=np.int64)
    for r in range(T):
        got = o.slice_qkv_heads(Wq, q["heads"], T, r)[:, 0]
        want = np.concatenate([np.arange(a, b) for a, b in q[str(r)]])
        assert np.array_equal(got, want)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 6, 12])
def test_colwise_shards_concatenate_to_weight(T):
    W = _rng(T).integers(0, 65535, size=(24, 10)).astype(np.uint16)
    shards = [o.slice_colwise(W, T, r) for r in range(T)]
    assert all(s.shape == (24 // T, 10) for s in shards)
    assert np.array_equal(np.concatenate(shards, axis=0), W)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 6, 12])
def test_rowwise_shards_interleave_to_weight(T):
    W = _rng(T).integers(0, 65535, size=(10, 24)).astype(np.uint16)
    shards = [o.slice_rowwise(W, T, r) for r in range(T)]
    assert all(s.shape == (10, 24 // T) for s in shards)
    assert np.array_equal(np.concatenate(shards, axis=1), W)


@pytest.mark.parametrize("heads,T", [(1, 1), (2, 2), (4, 2), (4, 4), (6, 3), (8, 8)])
def test_qkv_head_split_is_exact_partition(heads, T):
    D = heads * o.HEAD_DIM
    rows = np.arange(3 * D)  # row i of W_qkv carries label i
    Wq = np.repeat(rows[:, None], D, axis=1).astype(np.int32)
    seen = []
    hs = heads // T
    for r in range(T):
        lab = o.slice_qkv_heads(Wq, heads, T, r)[:, 0]
        assert lab.shape == (3 * D // T,)
        for blk in range(3):  # Q, K, V order inside the shard
            part = lab[blk * hs * 128:(blk + 1) * hs * 128]
            for j in range(hs):
                h = r * hs + j  # global head index
                want = blk * D + h * 128 + np.arange(128)
                assert np.array_equal(part[j * 128:(j + 1) * 128], want)
        seen.append(lab)
    allrows = np.sort(np.concatenate(seen))
    assert np.array_equal(allrows, rows)  # every row exactly once


def test_constraint_checks():
    W = np.zeros((12, 8))
    with pytest.raises(ValueError):
        o.slice_colwise(W, 5, 0)
    with pytest.raises(ValueError):
        o.slice_rowwise(W, 3, 0)
    with pytest.raises(ValueError):
        o.slice_colwise(W, 0, 0)
    with pytest.raises(ValueError):
        o.slice_colwise(W, 2, 2)
    with pytest.raises(ValueError):
        o.slice_colwise(W, 2, -1)
    # every packed block must be divisible on its own, not only their sum
    with pytest.raises(ValueError):
        o.slice_packed_colwise(np.zeros((8, 2)), [2, 6], 4, 0)
    o.slice_packed_colwise(np.zeros((8, 2)), [4, 4], 4, 0)
    # the degree must divide the head count
    with pytest.raises(ValueError):
        o.slice_qkv_heads(np.zeros((3 * 384, 384)), 3, 2, 0)
    with pytest.raises(ValueError):
        o.check_heads(300, 3, 1)


# ---------------------------------------------------------------------------
# GEMM / linear: brute force on tiny shapes, identity pass-through, closed form.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n_out", [4, 5])  # 5: a square weight, where a transpose still runs
def test_linear_matches_triple_loop(n_out):
    rng = _rng(1)
    X = rng.standard_normal((3, 5))
    W = rng.standard_normal((n_out, 5))
    b = rng.standard_normal(n_out)
    Y = o.linear(X, W, b)
    for i in range(3):
        for j in range(n_out):
            acc = b[j]
            for k in range(5):
                acc += X[i, k] * W[j, k]
            assert abs(Y[i, j] - acc) < 1e-12


def test_linear_identity_and_single_entry():
    X = _rng(2).standard_normal((6, 7))
    assert np.array_equal(o.linear(X, np.eye(7)), X)
    W = np.zeros((3, 7))
    W[2, 4] = 2.5
    Y = o.linear(X, W)
    assert np.array_equal(Y[:, 2], 2.5 * X[:, 4])
    assert np.all(Y[:, :2] == 0)


# ---------------------------------------------------------------------------
# GELU (tanh form): special values and the exact erf GELU within the tanh form's
# known approximation error.
# ---------------------------------------------------------------------------

def test_gelu_special_values():
    g = o.gelu_tanh
    assert g(np.array([0.0]))[0] == 0.0
    assert abs(g(np.array([12.0]))[0] - 12.0) < 1e-12
    assert abs(g(np.array([-12.0]))[0]) < 1e-12
    x = np.linspace(-6, 6, 1001)
    assert np.allclose(g(-x), g(x) - x, atol=1e-13)  # odd part of GELU is x/2
    # derivative at 0 is 1/2
    h = 1e-6
    assert abs((g(np.array([h]))[0] - g(np.array([-h]))[0]) / (2 * h) - 0.5) < 1e-8


def test_gelu_close_to_erf_gelu():
    x = np.linspace(-8, 8, 40001)
    exact = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in x])
    # the tanh form stays within 5e-4 of x*Phi(x) (max gap about 4.7e-4 near |x| = 2.7)
    assert np.max(np.abs(o.gelu_tanh(x) - exact)) < 5e-4


# ---------------------------------------------------------------------------
# Softmax / SDPA: closed forms and brute force.
# ---------------------------------------------------------------------------

def test_sdpa_equal_keys_gives_mean_of_values():
    rng = _rng(3)
    Q = rng.standard_normal((5, 128))
    K = np.tile(rng.standard_normal((1, 128)), (9, 1))
    V = rng.standard_normal((9, 128))
    O = o.sdpa(Q, K, V)
    assert np.allclose(O, np.tile(V.mean(axis=0), (5, 1)), atol=1e-13)


def test_sdpa_single_key_and_dominant_key():
    rng = _rng(4)
    Q = rng.standard_normal((4, 128))
    V = rng.standard_normal((1, 128))
    assert np.allclose(o.sdpa(Q, rng.standard_normal((1, 128)), V), np.tile(V, (4, 1)), atol=1e-14)
    q = rng.standard_normal((1, 128))
    K = rng.standard_normal((6, 128)) * 0.01
    K[3] = 400.0 * q[0] / np.linalg.norm(q)
    V = rng.standard_normal((6, 128))
    assert np.allclose(o.sdpa(q, K, V), V[3:4], atol=1e-9)


def test_sdpa_scale_closed_form():
    # q.k0 / sqrt(128) = ln 3 and q.k1 = 0  =>  weights 3/4 and 1/4.
    q = np.zeros((1, 128))
    q[0, 0] = math.sqrt(128.0) * math.log(3.0)
    K = np.zeros((2, 128))
    K[0, 0] = 1.0
    V = _rng(5).standard_normal((2, 128))
    assert np.allclose(o.sdpa(q, K, V), 0.75 * V[0] + 0.25 * V[1], atol=1e-14)


def test_sdpa_matches_scalar_loops():
    rng = _rng(6)
    Q = rng.standard_normal((3, 128))
    K = rng.standard_normal((4, 128))
    V = rng.standard_normal((4, 128))
    O = o.sdpa(Q, K, V)
    for i in range(3):
        s = [sum(Q[i, c] * K[j, c] for c in range(128)) / math.sqrt(128) for j in range(4)]
        e = [math.exp(v) for v in s]  # no max subtraction here: values are small
        z = sum(e)
        for c in range(0, 128, 17):
            want = sum(e[j] / z * V[j, c] for j in range(4))
            assert abs(O[i, c] - want) < 1e-12


def test_softmax_rows_sum_to_one_and_shift_invariant():
    S = _rng(7).standard_normal((5, 33)) * 30
    P = o.softmax_rows(S)
    assert np.allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert np.allclose(o.softmax_rows(S + 1000.0), P, atol=1e-14)


# ---------------------------------------------------------------------------
# The TP identities the pages state: sharded-then-summed == unsharded.
# ---------------------------------------------------------------------------

def _int_mlp(M, D, F, seed):
    rng = _rng(seed)
    return (rng.integers(-2, 3, size=(M, D)).astype(np.float64),
            rng.integers(-2, 3, size=(F, D)).astype(np.float64),
            rng.integers(-2, 3, size=F).astype(np.float64),
            rng.integers(-2, 3, size=(D, F)).astype(np.float64),
            rng.integers(-2, 3, size=D).astype(np.float64))


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_mlp_sharded_equals_unsharded_exactly_on_integers(T):
    X, Wu, bu, Wd, bd = _int_mlp(6, 16, 32, T)
    ident = lambda x: x  # noqa: E731  (integer sums stay exact in fp64)
    full = o.mlp_unsharded(X, Wu, bu, Wd, bd, act=ident)
    assert np.array_equal(o.mlp_sharded_summed(X, Wu, bu, Wd, bd, T, act=ident), full)


def test_mlp_closed_form_on_integers():
    # identity activation: Y = (X Wu^T + bu) Wd^T + bd, written as explicit loops.
    X, Wu, bu, Wd, bd = _int_mlp(2, 3, 4, 11)
    ident = lambda x: x  # noqa: E731
    Y = o.mlp_sharded_summed(X, Wu, bu, Wd, bd, 2, act=ident)
    for i in range(2):
        for j in range(3):
            h = [sum(X[i, k] * Wu[f, k] for k in range(3)) + bu[f] for f in range(4)]
            assert Y[i, j] == sum(h[f] * Wd[j, f] for f in range(4)) + bd[j]


@pytest.mark.parametrize("T", [1, 2, 4])
def test_mlp_sharded_equals_unsharded_with_gelu(T):
    d = syn.mlp_inputs(8, 128, 256, seed=9)
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items()}
    full = o.mlp_unsharded(f["X"], f["W_up"], f["b_up"], f["W_down"], f["b_down"])
    tp = o.mlp_sharded_summed(f["X"], f["W_up"], f["b_up"], f["W_down"], f["b_down"], T)
    assert np.max(np.abs(tp - full)) <= 1e-12 * np.max(np.abs(full))


def test_colwise_concatenation_is_full_hidden():
    d = syn.mlp_inputs(8, 128, 256, seed=10)
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items()}
    H = o.gelu_tanh(o.linear(f["X"], f["W_up"], f["b_up"]))
    Hs = np.concatenate([o.mlp_colwise_shard(f["X"], f["W_up"], f["b_up"], 4, r) for r in range(4)], axis=1)
    assert np.max(np.abs(Hs - H)) <= 1e-13 * np.max(np.abs(H))


def test_reduce_partials_sum_and_single_bias():
    parts = [np.full((2, 3), float(r + 1)) for r in range(4)]
    b = np.array([10.0, 20.0, 30.0])
    Y = o.reduce_partials(parts, b)
    assert np.array_equal(Y, np.tile(np.array([20.0, 30.0, 40.0]), (2, 1)))  # 1+2+3+4 + b


@pytest.mark.parametrize("heads,T", [(2, 1), (2, 2), (4, 2), (4, 4)])
def test_attention_sharded_equals_unsharded(heads, T):
    D = heads * 128
    d = syn.attn_inputs(24, D, seed=heads * 10 + T)
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items()}
    full = o.attn_unsharded(f["X"], f["W_qkv"], f["W_o"], heads)
    tp = o.attn_sharded_summed(f["X"], f["W_qkv"], f["W_o"], heads, T)
    assert np.max(np.abs(tp - full)) <= 1e-12 * np.max(np.abs(full))


def test_attention_zero_queries_closed_form():
    # W_q = 0 makes every score 0: each head averages its V over all tokens, so with
    # W_o = I the output row is mean_tokens(X) W_v^T for every query.  Swapping the
    # K and V blocks, or misreading the head layout, breaks this.
    heads, M = 2, 7
    D = heads * 128
    rng = _rng(12)
    X = rng.standard_normal((M, D))
    Wk = rng.standard_normal((D, D))
    Wv = rng.standard_normal((D, D))
    Wqkv = np.concatenate([np.zeros((D, D)), Wk, Wv], axis=0)
    Y = o.attn_unsharded(X, Wqkv, np.eye(D), heads)
    want = X.mean(axis=0) @ Wv.T
    assert np.allclose(Y, np.tile(want, (M, 1)), atol=1e-11)
    Y2 = o.attn_sharded_summed(X, Wqkv, np.eye(D), heads, 2)
    assert np.allclose(Y2, Y, atol=1e-11)


def test_attention_head_locality():
    # Head h's output depends only on head h's Q/K/V columns: zero every Q/K/V row of
    # head 1 except V's, and head 1's output becomes the token mean of its V, while
    # head 0 is unchanged.
    heads, M = 2, 9
    D = heads * 128
    rng = _rng(13)
    X = rng.standard_normal((M, D))
    W = rng.standard_normal((3 * D, D)) / np.sqrt(D)
    W2 = W.copy()
    W2[128:256] = 0.0           # Q of head 1
    W2[D + 128:D + 256] = 0.0   # K of head 1
    I = np.eye(D)
    A = o.attn_unsharded(X, W, I, heads)
    B = o.attn_unsharded(X, W2, I, heads)
    assert np.allclose(A[:, :128], B[:, :128], atol=1e-12)
    Vh1 = X @ W[2 * D + 128:2 * D + 256].T
    assert np.allclose(B[:, 128:], np.tile(Vh1.mean(axis=0), (M, 1)), atol=1e-12)


def test_attn_rows_match_full():
    heads = 2
    d = syn.attn_inputs(20, heads * 128, seed=14)
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items()}
    full = o.attn_sharded_summed(f["X"], f["W_qkv"], f["W_o"], heads, 2)
    rows = [0, 7, 19]
    part = o.attn_rows(f["X"], f["W_qkv"], f["W_o"], heads, rows, tp_degree=2)
    assert np.allclose(part, full[rows], rtol=0, atol=1e-12)


def test_round_bf16_values():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3])
    got = o.round_bf16(x)
    # ties to even at 1 + 2^-8 (halfway between 1 and 1 + 2^-7), up at 1 + 3*2^-8
    assert list(got[:4]) == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]
    assert abs(got[4] - 1e-3) <= 1e-3 * 2 ** -8


# ---------------------------------------------------------------------------
# Planted mistakes: every one must be caught by a pin above (run on the CPU).
# ---------------------------------------------------------------------------

def _run_pins():
    """Run a selection of pins; return the names of the ones that fail."""
    pins = {
        "fixture": test_slices_match_hand_fixture,
        "colcat": lambda: test_colwise_shards_concatenate_to_weight(4),
        "rowcat": lambda: test_rowwise_shards_interleave_to_weight(4),
        "qkv": lambda: test_qkv_head_split_is_exact_partition(4, 2),
        "loop": lambda: test_linear_matches_triple_loop(4),
        "loop_square": lambda: test_linear_matches_triple_loop(5),
        "gelu_erf": test_gelu_close_to_erf_gelu,
        "scale": test_sdpa_scale_closed_form,
        "mlp_int": lambda: test_mlp_sharded_equals_unsharded_exactly_on_integers(4),
        "mlp_closed": test_mlp_closed_form_on_integers,
        "mlp_gelu": lambda: test_mlp_sharded_equals_unsharded_with_gelu(2),
        "softmax": test_softmax_rows_sum_to_one_and_shift_invariant,
        "zero_q": test_attention_zero_queries_closed_form,
        "locality": test_attention_head_locality,
    }
    failed = []
    for name, fn in pins.items():
        try:
            fn()
        except Exception:  # noqa: BLE001 - any failure counts
            failed.append(name)
    return failed


def test_pins_pass_unmodified():
    assert _run_pins() == []


# Each planted mistake is a one-place edit of the oracle's C++ source: the
# test compiles the edited copy into its own library and runs the pins on it.
MUTANTS = {
    "bias_per_shard": ("Y[i * N + j] = bias ? acc + bias[j] : acc;",
                       "Y[i * N + j] = bias ? acc + T * bias[j] : acc;"),
    "bias_dropped": ("Y[(g * R + r) * N + j0 + q] = b ? acc[q][r] + b[j0 + q] : acc[q][r];",
                     "Y[(g * R + r) * N + j0 + q] = acc[q][r];"),
    "transposed": ("const double wk = w[q][k];", "const double wk = W[k * N + j0 + (q < nj ? q : 0)];"),
    "colwise_off_by_one": ("std::memcpy(out, W + r * step * cols * es, size_t(step * cols * es));",
                           "std::memcpy(out, W + ((r + 1) % T) * step * cols * es, size_t(step * cols * es));"),
    "rowwise_strided": ("std::memcpy(out + i * step * es, W + (i * cols + r * step) * es, size_t(step * es));",
                        "for (int64_t c = 0; c < step; ++c) "
                        "std::memcpy(out + (i * step + c) * es, W + (i * cols + r + c * T) * es, size_t(es));"),
    "gelu_coeff": ("0.044715 * x * x * x", "0.04715 * x * x * x"),
    "scale_missing": ("for (int64_t t = 0; t < n * Mk; ++t) S[size_t(t)] *= scale;", ""),
    "qkv_interleaved": ("return slice_packed_colwise(W, rows, D, es, blocks, 3, T, r, out);",
                        "return slice_colwise(W, rows, D, es, T, r, out);"),
    "activation_skipped": ("  apply_act(H, M * (F / T), act);\n  return kOk;", "  return kOk;"),
    "softmax_unnormalised": ("for (int64_t j = 0; j < cols; ++j) p[j] /= l;", ""),
}


@pytest.fixture(scope="module")
def mutant_libs(tmp_path_factory):
    """Every mutant compiled once (in parallel) from an edited copy of oracle.cpp."""
    from concurrent.futures import ThreadPoolExecutor

    from oracle import build as ob
    src = open(ob.SRC).read()
    out = tmp_path_factory.mktemp("oracle_mutants")

    def one(item):
        name, (old, new) = item
        assert src.count(old) == 1, f"mutant {name}: the edited text must occur exactly once"
        return name, ob.compile_source(src.replace(old, new), str(out / f"lib_{name}.so"))

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return dict(ex.map(one, MUTANTS.items()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_have_teeth(name, mutant_libs):
    with o.using_library(mutant_libs[name]):
        assert _run_pins() != [], f"planted mistake {name!r} was not caught by any pin"


# ---------------------------------------------------------------------------
# The seeded generator (shared input module).
# ---------------------------------------------------------------------------

def test_generator_deterministic_and_distinct_streams():
    a = syn.normal_bf16((1000,), 1.0, seed=1, tid=0)
    b = syn.normal_bf16((1000,), 1.0, seed=1, tid=0)
    c = syn.normal_bf16((1000,), 1.0, seed=1, tid=1)
    d = syn.normal_bf16((1000,), 1.0, seed=2, tid=0)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # a prefix of a longer draw is the shorter draw (element i depends only on i)
    e = syn.normal_bf16((3000,), 1.0, seed=1, tid=0)
    assert np.array_equal(e[:1000], a)


def test_generator_statistics():
    x = syn.bf16_bits_to_f64(syn.normal_bf16((1 << 20,), 0.5, seed=3, tid=4))
    assert abs(x.mean()) < 3e-3
    assert abs(x.std() / 0.5 - 1) < 5e-3
    assert abs(np.mean(np.abs(x) < 0.5) - 0.6827) < 3e-3  # one-sigma mass of a normal


def test_bf16_encoding():
    v = np.array([1.0, -2.0, 0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32)
    bits = syn._f32_to_bf16_bits(v)
    assert list(bits) == [0x3F80, 0xC000, 0x0000, 0x3F80, 0x3F82]
    assert np.array_equal(syn.bf16_bits_to_f64(bits), np.array([1.0, -2.0, 0.0, 1.0, 1.0 + 2 ** -6]))


def test_block_rows_returns_exact_attention_and_mlp_of_rounded_input():
    heads, M, D, F = 2, 12, 256, 512
    d = syn.block_inputs(M, D, F, seed=21)
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items()}
    rows = [0, 5, 11]
    A, Y = o.block_rows(f["X"], f["W_qkv"], f["W_o"], heads, f["W_up"], f["b_up"], f["W_down"], f["b_down"],
                        rows, tp_degree=2)
    A_full = o.attn_unsharded(f["X"], f["W_qkv"], f["W_o"], heads)
    assert np.allclose(A, A_full[rows], atol=1e-12)
    Y_want = o.mlp_unsharded(o.round_bf16(A_full[rows]), f["W_up"], f["b_up"], f["W_down"], f["b_down"])
    assert np.allclose(Y, Y_want, atol=1e-12)


# ---------------------------------------------------------------------------
# Packed styles, SwiGLU pair, rowwise_split_input ("Fused projections" and the
# style table's third row).
# ---------------------------------------------------------------------------

def test_packed_fixtures():
    g = json.load(open(GOLDEN))
    f = g["packed_colwise_fused_qkv_gate_up"]
    W = np.arange(f["rows"])[:, None] * np.ones((1, 2), dtype=np.int64)
    for r in range(f["tp_degree"]):
        assert list(o.slice_packed_colwise(W, f["blocks"], f["tp_degree"], r)[:, 0]) == f[str(r)]
    f = g["packed_rowwise_absolute"]
    W = np.arange(f["cols"])[None, :]
    for r in range(f["tp_degree"]):
        assert list(o.slice_packed_rowwise(W, f["blocks"], f["tp_degree"], r)[0]) == f[str(r)]


def test_packed_block_rules():
    assert o.packed_block_sizes(36, [1, 1, 1, 3, 3], 2) == [4, 4, 4, 12, 12]
    assert o.packed_block_sizes(12, [4, 8], 2) == [4, 8]         # absolute sizes
    assert o.packed_block_sizes(12, [1, 2], 2) == [4, 8]         # proportional form of the same
    with pytest.raises(ValueError):
        o.packed_block_sizes(10, [1, 2], 1)                      # sum 3 does not divide 10
    with pytest.raises(ValueError):
        o.packed_block_sizes(18, [1, 1, 1, 3, 3], 3)             # blocks 2,2,2,6,6: 2 % 3 != 0
    assert o.packed_block_sizes(12, [2, 1], 4) == [8, 4]         # each block divisible
    with pytest.raises(ValueError):
        o.packed_block_sizes(12, [5, 1], 4)                      # 10, 2: the sum 12 is divisible, the blocks are not


def test_packed_equals_plain_for_one_block():
    W = _rng(30).integers(0, 9, size=(12, 8))
    for r in range(4):
        assert np.array_equal(o.slice_packed_colwise(W, [1], 4, r), o.slice_colwise(W, 4, r))
        assert np.array_equal(o.slice_packed_rowwise(W, [1], 4, r), o.slice_rowwise(W, 4, r))


def test_silu_values():
    x = np.array([0.0, 1.0, -1.0, 20.0, -20.0])
    want = np.array([0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1)), 20 / (1 + math.exp(-20)),
                     -20 / (1 + math.exp(20))])
    assert np.allclose(o.silu(x), want, rtol=1e-15, atol=1e-300)
    assert abs(o.silu(np.array([20.0]))[0] - 20.0) < 1e-6


@pytest.mark.parametrize("T", [1, 2, 4])
def test_swiglu_sharded_equals_unsharded(T):
    rng = _rng(31 + T)
    M, D, F = 5, 16, 32
    X = rng.standard_normal((M, D))
    W_in = rng.standard_normal((2 * F, D)) / 4
    b_in = rng.standard_normal(2 * F) * 0.1
    W_out = rng.standard_normal((D, F)) / 6
    b_out = rng.standard_normal(D) * 0.1
    full = o.swiglu_unsharded(X, W_in, b_in, W_out, b_out)
    tp = o.swiglu_sharded_summed(X, W_in, b_in, W_out, b_out, T)
    assert np.max(np.abs(tp - full)) <= 1e-12 * np.max(np.abs(full))


def test_swiglu_closed_form():
    # gate rows = 0 -> silu(0) = 0 -> output = b_out; up irrelevant.
    rng = _rng(33)
    M, D, F = 3, 8, 8
    X = rng.standard_normal((M, D))
    W_in = np.concatenate([np.zeros((F, D)), rng.standard_normal((F, D))])
    b_out = rng.standard_normal(D)
    Y = o.swiglu_sharded_summed(X, W_in, None, rng.standard_normal((D, F)), b_out, 2)
    assert np.allclose(Y, np.tile(b_out, (M, 1)), atol=1e-14)
    # gate = large positive constant c -> silu(c) ~ c, so H ~ c * up
    c = 30.0
    W_g = np.zeros((F, D))
    b_in = np.concatenate([np.full(F, c), np.zeros(F)])
    W_u = rng.standard_normal((F, D))
    W_out = rng.standard_normal((D, F))
    Y = o.swiglu_sharded_summed(X, np.concatenate([W_g, W_u]), b_in, W_out, None, 2)
    assert np.allclose(Y, c * (X @ W_u.T) @ W_out.T, rtol=1e-9)


@pytest.mark.parametrize("T", [1, 2, 3, 6])
def test_rowwise_split_input_is_the_full_projection(T):
    rng = _rng(40 + T)
    X = rng.integers(-3, 4, size=(4, 12)).astype(np.float64)
    W = rng.integers(-3, 4, size=(7, 12)).astype(np.float64)
    b = rng.integers(-3, 4, size=7).astype(np.float64)
    assert np.array_equal(o.rowwise_split_input(X, W, b, T), X @ W.T + b)


# ---------------------------------------------------------------------------
# Dual-stream joint attention (image stream + text stream, one joint SDPA).
# ---------------------------------------------------------------------------

def _joint_inputs(seed, Mi=6, Mt=3, D=256):
    rng = _rng(seed)
    w = lambda *s: rng.standard_normal(s) / np.sqrt(s[-1])  # noqa: E731
    return (rng.standard_normal((Mi, D)), rng.standard_normal((Mt, D)), w(3 * D, D), w(3 * D, D), w(D, D),
            w(D, D))


def test_joint_with_shared_weights_is_attention_over_the_concatenation():
    Xi, Xt, Wq, _, Wo, _ = _joint_inputs(50)
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt, Wq, Wq, Wo, Wo, heads=2)
    Y = o.attn_unsharded(np.concatenate([Xi, Xt]), Wq, Wo, heads=2)
    assert np.allclose(np.concatenate([Yi, Yt]), Y, rtol=1e-13, atol=1e-13)


def test_joint_without_text_is_the_image_attention():
    Xi, Xt, Wqi, Wqt, Woi, Wot = _joint_inputs(51)
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt[:0], Wqi, Wqt, Woi, Wot, heads=2)
    assert Yt.shape == (0, Xi.shape[1])
    assert np.allclose(Yi, o.attn_unsharded(Xi, Wqi, Woi, heads=2), rtol=1e-13, atol=1e-13)


def test_joint_uniform_scores_average_both_streams():
    # Q = 0 in both streams: every score is 0, so each query averages V over ALL
    # joint tokens.  Attending each stream on its own would average per stream.
    Xi, Xt, Wqi, Wqt, Woi, Wot = _joint_inputs(52)
    D = Xi.shape[1]
    Wqi[:D] = 0
    Wqt[:D] = 0
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt, Wqi, Wqt, Woi, Wot, heads=2)
    V = np.concatenate([Xi @ Wqi[2 * D:].T, Xt @ Wqt[2 * D:].T])
    vbar = V.mean(axis=0)
    assert np.allclose(Yi, np.tile(vbar @ Woi.T, (Xi.shape[0], 1)), rtol=1e-12, atol=1e-12)
    assert np.allclose(Yt, np.tile(vbar @ Wot.T, (Xt.shape[0], 1)), rtol=1e-12, atol=1e-12)
    # the per-stream average differs, so this pin separates the two readings
    assert not np.allclose(V[:Xi.shape[0]].mean(axis=0), vbar)


def test_joint_token_order_does_not_matter():
    Xi, Xt, Wqi, Wqt, Woi, Wot = _joint_inputs(53)
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt, Wqi, Wqt, Woi, Wot, heads=2)
    Yt2, Yi2 = o.joint_attn_unsharded(Xt, Xi, Wqt, Wqi, Wot, Woi, heads=2)
    assert np.allclose(Yi, Yi2, rtol=1e-12, atol=1e-13) and np.allclose(Yt, Yt2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T", [1, 2])
def test_joint_sharded_equals_unsharded_and_rows(T):
    Xi, Xt, Wqi, Wqt, Woi, Wot = _joint_inputs(54 + T)
    Yi, Yt = o.joint_attn_unsharded(Xi, Xt, Wqi, Wqt, Woi, Wot, heads=2)
    Si, St = o.joint_attn_sharded_summed(Xi, Xt, Wqi, Wqt, Woi, Wot, 2, T)
    assert np.allclose(Si, Yi, rtol=1e-12, atol=1e-12) and np.allclose(St, Yt, rtol=1e-12, atol=1e-12)
    Ri, Rt = o.joint_attn_rows(Xi, Xt, Wqi, Wqt, Woi, Wot, 2, [0, 5], [2], tp_degree=T)
    assert np.allclose(Ri, Yi[[0, 5]], rtol=1e-12, atol=1e-12) and np.allclose(Rt, Yt[[2]], rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        o.joint_attn_sharded_summed(Xi, Xt, Wqi, Wqt, Woi, Wot, 2, 4)  # 4 does not divide 2 heads


# ---------------------------------------------------------------------------
# Context parallelism ("Context parallelism" page): Ring attention's merge of
# per-key-block results and Ulysses attention's head regrouping.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("splits", [[7], [3, 4], [1, 2, 4], [2, 2, 2, 1]])
def test_ring_merge_of_key_blocks_is_attention_over_all_keys(splits):
    rng = _rng(60 + len(splits))
    Mq, d = 5, 16
    Mk = sum(splits)
    Q, K, V = rng.standard_normal((Mq, d)), rng.standard_normal((Mk, d)), rng.standard_normal((Mk, d))
    full, lse_full = o.sdpa(Q, K, V, return_lse=True)
    parts, lses, j = [], [], 0
    for n in splits:
        Ob, lb = o.sdpa(Q, K[j:j + n], V[j:j + n], scale=1 / np.sqrt(d), return_lse=True)
        parts.append(Ob)
        lses.append(lb)
        j += n
    O, lse = o.attn_merge(np.stack(parts), np.stack(lses))
    assert np.max(np.abs(O - full)) <= 1e-12 and np.max(np.abs(lse - lse_full)) <= 1e-12
    # the merge does not depend on the order the blocks arrive in (ranks see them rotated)
    O2, _ = o.attn_merge(np.stack(parts[::-1]), np.stack(lses[::-1]))
    assert np.max(np.abs(O2 - full)) <= 1e-12


def test_lse_closed_form():
    # one key per block: lse = s * scale; equal scores: lse = log(Mk) + s
    Q = np.array([[1.0, 2.0]])
    K = np.array([[3.0, -1.0], [3.0, -1.0], [3.0, -1.0]])
    V = np.eye(3, 2)
    _, lse = o.sdpa(Q, K, V, scale=0.5, return_lse=True)
    assert abs(lse[0] - (np.log(3.0) + 0.5 * 1.0)) <= 1e-14
    # a block with much smaller weight barely moves the merge
    O, _ = o.attn_merge(np.array([[[1.0, 0.0]], [[0.0, 1.0]]]), np.array([[0.0], [np.log(3.0)]]))
    assert np.allclose(O, [[0.25, 0.75]], atol=1e-15)


def test_ulysses_regrouping_is_attention_over_all_tokens():
    # U ranks hold M/U tokens with all H heads; packing each rank's [Q|K|V] by
    # destination head group (packed rowwise, blocks [1, 1, 1]), exchanging
    # (all-to-all), attending all tokens x H/U heads and regrouping back must
    # give the full attention -- exactly, since every head sees the same data.
    rng = _rng(70)
    U, H, d, M = 2, 4, 8, 6
    QKV = rng.standard_normal((M, 3 * H * d))
    def attend(qkv, n_heads):
        c = n_heads * d
        return np.concatenate([o.sdpa(qkv[:, h * d:(h + 1) * d], qkv[:, c + h * d:c + (h + 1) * d],
                                      qkv[:, 2 * c + h * d:2 * c + (h + 1) * d]) for h in range(n_heads)], axis=1)
    full = attend(QKV, H)
    Ms = M // U
    send = [[o.slice_packed_rowwise(QKV[s * Ms:(s + 1) * Ms], [1, 1, 1], U, u) for u in range(U)] for s in range(U)]
    out_blocks = []
    for u in range(U):  # rank u receives every rank's tokens for head group u, in rank (= token) order
        O_u = attend(np.concatenate([send[s][u] for s in range(U)]), H // U)
        out_blocks.append(O_u)
    got = np.concatenate([np.concatenate([out_blocks[u][s * Ms:(s + 1) * Ms] for u in range(U)], axis=1)
                          for s in range(U)])
    assert np.array_equal(got, full)
