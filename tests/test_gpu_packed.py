"""Packed styles, the SwiGLU pair and rowwise_split_input on the GPU against
the fp64 oracle ("Fused projections" section and the style table's third row
of the Diffusers "Tensor parallelism" page).

* packed colwise / rowwise slicing is bit-exact against the oracle's slices,
  for proportional blocks ([1, 1, 1, 3, 3], [1, 1]) and absolute sizes;
* the SwiGLU colwise GEMM (gate and up in one accumulator tile) and the
  SwiGLU pair, on ragged shapes through both GEMM kernels and on the
  Flux-scale shape with mlp_ratio 3;
* rowwise_split_input, whose input slice is a TMA coordinate into the
  replicated input, including K/T not a multiple of the 64-wide K block;
* a packed rowwise output projection (absolute blocks [inner_dim,
  mlp_hidden_dim]) fed with per-shard [attention | MLP] activations equals
  the unsharded projection of the concatenation.
"""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, assert_rounded_once, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _dev(d):
    return {k: to_dev(v) for k, v in d.items()}


def _empty(shape):
    return torch.full(shape, 0x7FC1, dtype=torch.int16, device="cuda")  # a NaN pattern: unwritten shows


# --------------------------------------------------------------------------- slicing
@pytest.mark.parametrize("rows,cols,blocks,T", [
    (9 * 256, 256, [1, 1, 1, 3, 3], 2),   # fused Q, K, V, gate, up with mlp_ratio 3 (D = 256)
    (9 * 256, 256, [1, 1, 1, 3, 3], 4),
    (2 * 1024, 64, [1, 1], 8),            # SwiGLU gate/up halves
    (2 * 1024, 64, [1024, 1024], 8),      # the same as absolute sizes
    (1200, 40, [3, 1, 2], 4),             # uneven proportions, rows of 80 bytes
])
def test_packed_colwise_bit_exact(rows, cols, blocks, T):
    W = syn.normal_bf16((rows, cols), 1.0, seed=rows + T, tid=400)
    Wd = to_dev(W)
    allout = _empty((T, rows // T, cols))
    assert tp.tp_shard_packed_all(Wd, rows, cols, tp.TP_COLWISE, blocks, T, allout) == 0
    for r in range(T):
        one = _empty((rows // T, cols))
        assert tp.tp_shard_packed(Wd, rows, cols, tp.TP_COLWISE, blocks, T, r, one) == 0
        torch.cuda.synchronize()
        want = o.slice_packed_colwise(W, blocks, T, r)
        assert np.array_equal(from_dev(one), want)
        assert np.array_equal(from_dev(allout[r]), want)


@pytest.mark.parametrize("rows,cols,blocks,T", [
    (64, 256 + 768, [256, 768], 4),       # absolute [inner_dim, mlp_hidden_dim]
    (64, 256 + 768, [1, 3], 4),           # the same, proportional
    (1, 2 * 512, [1, 1], 2),              # a packed colwise bias, sliced as a 1 x n matrix
    (33, 9 * 64, [1, 1, 1, 3, 3], 8),     # shard widths 8, 8, 8, 24, 24
])
def test_packed_rowwise_bit_exact(rows, cols, blocks, T):
    W = syn.normal_bf16((rows, cols), 1.0, seed=cols + T, tid=401)
    Wd = to_dev(W)
    allout = _empty((T, rows, cols // T))
    assert tp.tp_shard_packed_all(Wd, rows, cols, tp.TP_ROWWISE, blocks, T, allout) == 0
    for r in range(T):
        one = _empty((rows, cols // T))
        assert tp.tp_shard_packed(Wd, rows, cols, tp.TP_ROWWISE, blocks, T, r, one) == 0
        torch.cuda.synchronize()
        want = o.slice_packed_rowwise(W, blocks, T, r)
        assert np.array_equal(from_dev(one), want)
        assert np.array_equal(from_dev(allout[r]), want)


def test_packed_with_one_block_is_the_plain_slice():
    W = syn.normal_bf16((512, 128), 1.0, seed=9, tid=402)
    Wd = to_dev(W)
    a, b = _empty((4, 128, 128)), _empty((4, 128, 128))
    assert tp.tp_shard_packed_all(Wd, 512, 128, tp.TP_COLWISE, [1], 4, a) == 0
    assert tp.tp_shard_weight_all(Wd, 512, 128, tp.TP_COLWISE, 4, b) == 0
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(a), from_dev(b))


def test_shard_batch_mixed_jobs_bit_exact():
    # plain colwise, plain rowwise, a bias, packed colwise [1,1,1,3,3] and packed
    # rowwise [256, 768] in one call: 1 + 1 + 1 + 5 + 2 = 10 copy jobs, one launch.
    T = 4
    Wc = syn.normal_bf16((512, 136), 1.0, seed=1, tid=440)
    Wr = syn.normal_bf16((72, 1024), 1.0, seed=2, tid=441)
    b = syn.normal_bf16((2048,), 1.0, seed=3, tid=442)
    Wpc = syn.normal_bf16((9 * 128, 64), 1.0, seed=4, tid=443)
    Wpr = syn.normal_bf16((40, 1024), 1.0, seed=5, tid=444)
    outs = [_empty((T, 128, 136)), _empty((T, 72, 256)), _empty((T, 512)), _empty((T, 9 * 32, 64)),
            _empty((T, 40, 256))]
    jobs = [(to_dev(Wc), 512, 136, tp.TP_COLWISE, outs[0]), (to_dev(Wr), 72, 1024, tp.TP_ROWWISE, outs[1]),
            (to_dev(b), T, 512, tp.TP_COLWISE, outs[2]),
            (to_dev(Wpc), 9 * 128, 64, tp.TP_COLWISE, outs[3], [1, 1, 1, 3, 3]),
            (to_dev(Wpr), 40, 1024, tp.TP_ROWWISE, outs[4], [256, 768])]
    n0 = tp.tp_kernel_launches()
    assert tp.tp_shard_weights_batch(jobs, T) == 0
    assert tp.tp_kernel_launches() - n0 == 1
    torch.cuda.synchronize()
    for r in range(T):
        assert np.array_equal(from_dev(outs[0][r]), o.slice_colwise(Wc, T, r))
        assert np.array_equal(from_dev(outs[1][r]), o.slice_rowwise(Wr, T, r))
        assert np.array_equal(from_dev(outs[2][r]), o.slice_colwise(b, T, r))
        assert np.array_equal(from_dev(outs[3][r]), o.slice_packed_colwise(Wpc, [1, 1, 1, 3, 3], T, r))
        assert np.array_equal(from_dev(outs[4][r]), o.slice_packed_rowwise(Wpr, [256, 768], T, r))


# --------------------------------------------------------------------------- SwiGLU colwise GEMM
@pytest.mark.parametrize("M,K,Fs,T,bias", [
    (64, 128, 256, 2, True),     # one-CTA kernel
    (129, 72, 72, 3, True),      # ragged M, K and F_s < 128: gate tile reaches into the up rows
    (129, 72, 264, 3, False),    # ragged, three output tiles
    (257, 192, 264, 2, True),    # CTA-pair kernel, ragged
    (512, 256, 512, 4, True),    # CTA-pair kernel, whole tiles
])
def test_colwise_swiglu(M, K, Fs, T, bias):
    X = syn.normal_bf16((M, K), 1.0, seed=M, tid=410)
    W = syn.normal_bf16((T, 2 * Fs, K), 1.0 / np.sqrt(K), seed=K + Fs, tid=411)  # shard r = [gate_r; up_r]
    b = syn.normal_bf16((T, 2 * Fs), 0.5, seed=Fs, tid=412) if bias else None
    out = _empty((T, M, Fs))
    assert tp.tp_colwise_swiglu(to_dev(X), M, K, to_dev(W), to_dev(b) if bias else None, Fs, T, out) == 0
    torch.cuda.synchronize()
    g = from_dev(out)
    for r in range(T):
        G = o.linear(f64(X), f64(W[r, :Fs]), f64(b[r, :Fs]) if bias else None)
        U = o.linear(f64(X), f64(W[r, Fs:]), f64(b[r, Fs:]) if bias else None)
        assert_rounded_once(g[r], o.silu(G) * U, f"swiglu shard {r}")


# --------------------------------------------------------------------------- rowwise_split_input
@pytest.mark.parametrize("M,K,N,T,bias", [
    (64, 256, 128, 2, True),     # one-CTA kernel
    (129, 216, 264, 3, True),    # K/T = 72: shard slices end inside a 64-wide K block
    (257, 216, 264, 3, False),   # CTA-pair kernel, ragged
    (512, 1024, 520, 8, True),   # CTA-pair kernel, 8 shards walked by one accumulator
])
def test_rowwise_split_input(M, K, N, T, bias):
    X = syn.normal_bf16((M, K), 1.0, seed=M, tid=420)
    W = syn.normal_bf16((N, K), 1.0 / np.sqrt(K), seed=K, tid=421)
    b = syn.normal_bf16((N,), 0.02, seed=N, tid=422) if bias else None
    Wd = to_dev(W)
    W_sh = _empty((T, N, K // T))
    assert tp.tp_shard_weight_all(Wd, N, K, tp.TP_ROWWISE_SPLIT_INPUT, T, W_sh) == 0
    Y = _empty((M, N))
    assert tp.tp_rowwise_split_input_linear(to_dev(X), M, K, W_sh, N, to_dev(b) if bias else None, T, Y) == 0
    torch.cuda.synchronize()
    ref = o.rowwise_split_input(f64(X), f64(W), f64(b) if bias else None, T)
    assert_parity(from_dev(Y), ref, f"rowwise_split_input T={T}")


def test_split_input_equals_explicitly_sliced_input():
    # Slicing the input first and running the plain rowwise sum performs the same
    # fp32 operations in the same order: the results must be bit-identical.
    M, K, N, T = 300, 512, 256, 4
    X = syn.normal_bf16((M, K), 1.0, seed=3, tid=423)
    W = syn.normal_bf16((N, K), 1.0 / np.sqrt(K), seed=4, tid=424)
    Xd, Wd = to_dev(X), to_dev(W)
    W_sh = _empty((T, N, K // T))
    X_sh = _empty((T, M, K // T))
    assert tp.tp_shard_weight_all(Wd, N, K, tp.TP_ROWWISE, T, W_sh) == 0
    assert tp.tp_shard_weight_all(Xd, M, K, tp.TP_ROWWISE, T, X_sh) == 0
    Y1, Y2 = _empty((M, N)), _empty((M, N))
    assert tp.tp_rowwise_split_input_linear(Xd, M, K, W_sh, N, None, T, Y1) == 0
    assert tp.tp_rowwise_linear_sum(X_sh, M, K // T, W_sh, N, None, T, Y2) == 0
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(Y1), from_dev(Y2))


# --------------------------------------------------------------------------- packed rowwise output projection
def test_packed_rowwise_output_projection():
    # A fused output projection whose input is [attention output | MLP hidden]
    # (absolute blocks [inner_dim, mlp_hidden_dim]).  Shard r holds
    # [attn_r | mlp_r] and the packed rowwise slice of W; the sum over shards is
    # the unsharded projection of the concatenated input.
    M, inner, hidden, N, T = 257, 256, 768, 256, 4
    A_attn = syn.normal_bf16((M, inner), 1.0, seed=1, tid=430)
    A_mlp = syn.normal_bf16((M, hidden), 1.0, seed=2, tid=431)
    W = syn.normal_bf16((N, inner + hidden), 1.0 / 32, seed=3, tid=432)
    b = syn.normal_bf16((N,), 0.02, seed=4, tid=433)
    A = np.concatenate([A_attn, A_mlp], axis=1)
    A_sh = np.stack([o.slice_packed_rowwise(A, [inner, hidden], T, r) for r in range(T)])  # per-rank activations
    W_sh = _empty((T, N, (inner + hidden) // T))
    assert tp.tp_shard_packed_all(to_dev(W), N, inner + hidden, tp.TP_ROWWISE, [inner, hidden], T, W_sh) == 0
    Y = _empty((M, N))
    Ks = (inner + hidden) // T
    assert tp.tp_rowwise_linear_sum(to_dev(A_sh), M, Ks, W_sh, N, to_dev(b), T, Y) == 0
    torch.cuda.synchronize()
    assert_parity(from_dev(Y), o.linear(f64(A), f64(W), f64(b)), "packed rowwise out-projection")


# --------------------------------------------------------------------------- SwiGLU pair
def _swiglu_pair(dd, T):
    Y = tp.swiglu_mlp_pair(dd["X"], dd["W_in"], dd["b_in"], dd["W_out"], dd["b_out"], T)
    torch.cuda.synchronize()
    return from_dev(Y)


@pytest.mark.parametrize("M,D,F,T", [(64, 128, 512, 2), (129, 136, 216, 3), (300, 256, 1024, 4)])
def test_swiglu_pair_small(M, D, F, T):
    d = syn.swiglu_inputs(M, D, F, seed=M)
    f = {k: f64(v) for k, v in d.items()}
    g = _swiglu_pair(_dev(d), T)
    ref = o.swiglu_sharded_summed(f["X"], f["W_in"], f["b_in"], f["W_out"], f["b_out"], T)
    assert_parity(g, ref, f"swiglu pair M={M} D={D} F={F} T={T}")


@pytest.fixture(scope="module")
def flux_swiglu():
    c = syn.CONFIGS["flux_swiglu"]
    d = syn.swiglu_inputs(c["M"], c["D"], c["F"], c["seed"])
    f = {k: f64(v) for k, v in d.items()}
    ref = o.swiglu_unsharded(f["X"], f["W_in"], f["b_in"], f["W_out"], f["b_out"])
    return c, d, ref


def test_flux_swiglu_pair(flux_swiglu):
    c, d, ref = flux_swiglu
    g = _swiglu_pair(_dev(d), c["T"])
    assert_parity(g, ref, "flux swiglu T=4")


def test_swiglu_bench_step_matches_one_shot():
    # bench.py times the SwiGLU pair as its three step calls (one batched slice
    # launch, the SwiGLU colwise GEMM, the rowwise GEMM); same bits as the one-shot call.
    import bench
    wl = bench.SwigluWorkload(dict(kind="swiglu", M=300, D=256, F=1024, T=4, seed=11))
    d = wl.host_inputs(0)
    g = {k: to_dev(v) for k, v in d.items()}
    n0 = tp.tp_kernel_launches()
    for k in wl.kernels(tp, g, "cuda"):
        k.fn()
    assert tp.tp_kernel_launches() - n0 == 3
    torch.cuda.synchronize()
    one = _swiglu_pair(g, 4)
    assert np.array_equal(from_dev(wl.bufs["Y"]), one)


def test_swiglu_prepare_run_matches_one_shot(flux_swiglu):
    c, d, _ = flux_swiglu
    dd = _dev(d)
    one = _swiglu_pair(dd, c["T"])
    layer = tp.MlpPair(dd["W_in"], dd["b_in"], dd["W_out"], dd["b_out"], c["T"], activation="swiglu")
    for _ in range(2):
        Y = layer(dd["X"])
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(Y), one)
    layer.close()
    # degree 1 and 8 also match the unsharded oracle, and every degree performs
    # the same fp32 operations in the same order (F/T stays a multiple of 64)
    for T in (1, 8):
        assert np.array_equal(_swiglu_pair(dd, T), one), f"T={T} differs from T={c['T']}"
    assert tp.tp_check_device_error() == 0
