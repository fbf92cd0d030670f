"""The MLP pair (a1..a4) on the GPU against the fp64 oracle: the tiny and the
Flux-scale configurations, the degree sweep {1,2,4,8} on the Flux-scale shape
(each degree must equal the unsharded oracle), ragged token counts, and the
prepare/run path."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _dev(d):
    return {k: to_dev(v) for k, v in d.items()}


def _run_pair(dd, M, D, F, T):
    Y = tp.mlp_pair(dd["X"], dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T)
    torch.cuda.synchronize()
    return from_dev(Y)


@pytest.fixture(scope="module")
def tiny():
    c = syn.CONFIGS["tiny_mlp"]
    d = syn.mlp_inputs(c["M"], c["D"], c["F"], c["seed"])
    return c, d, {k: f64(v) for k, v in d.items()}


@pytest.fixture(scope="module")
def flux():
    c = syn.CONFIGS["flux_mlp"]
    d = syn.mlp_inputs(c["M"], c["D"], c["F"], c["seed"])
    f = {k: f64(v) for k, v in d.items()}
    ref = o.mlp_unsharded(f["X"], f["W_up"], f["b_up"], f["W_down"], f["b_down"])
    return c, d, ref


def test_tiny_mlp_pair(tiny):
    c, d, f = tiny
    g = _run_pair(_dev(d), c["M"], c["D"], c["F"], c["T"])
    ref = o.mlp_sharded_summed(f["X"], f["W_up"], f["b_up"], f["W_down"], f["b_down"], c["T"])
    assert_parity(g, ref, "tiny mlp")


@pytest.mark.parametrize("M", [1, 5, 127, 129, 200])
def test_ragged_tokens(tiny, M):
    c, d, f = tiny
    X = syn.normal_bf16((M, c["D"]), 1.0, seed=M, tid=0)
    dd = _dev({**d, "X": X})
    g = _run_pair(dd, M, c["D"], c["F"], c["T"])
    ref = o.mlp_unsharded(f64(X), f["W_up"], f["b_up"], f["W_down"], f["b_down"])
    assert_parity(g, ref, f"mlp M={M}")


def test_flux_mlp_pair(flux):
    c, d, ref = flux
    g = _run_pair(_dev(d), c["M"], c["D"], c["F"], c["T"])
    assert_parity(g, ref, "flux mlp T=4")


def test_degree_sweep_matches_unsharded_and_is_bit_identical(flux):
    c, d, ref = flux
    dd = _dev(d)
    outs = {}
    for T in (1, 2, 4, 8):
        outs[T] = _run_pair(dd, c["M"], c["D"], c["F"], T)
        assert_parity(outs[T], ref, f"sweep T={T}")
    # F/T is a multiple of the 64-wide K block for every T, and the rowwise
    # accumulator walks shards in ascending order, so every degree performs the
    # same fp32 operations in the same order.
    for T in (2, 4, 8):
        assert np.array_equal(outs[T], outs[1]), f"T={T} differs from T=1"


def test_prepare_run_matches_one_shot(tiny, flux):
    for c, d in ((tiny[0], tiny[1]), (flux[0], flux[1])):
        dd = _dev(d)
        one = _run_pair(dd, c["M"], c["D"], c["F"], c["T"])
        layer = tp.MlpPair(dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], c["T"])
        for _ in range(2):
            Y = layer(dd["X"])
            torch.cuda.synchronize()
            assert np.array_equal(from_dev(Y), one)
        layer.close()


def test_no_bias(tiny):
    c, d, f = tiny
    dd = _dev(d)
    Y = tp.mlp_pair(dd["X"], dd["W_up"], None, dd["W_down"], None, c["T"])
    torch.cuda.synchronize()
    ref = o.mlp_unsharded(f["X"], f["W_up"], None, f["W_down"], None)
    assert_parity(from_dev(Y), ref, "no bias")


def test_empty_input_writes_nothing(tiny):
    c, d, f = tiny
    dd = _dev(d)
    Y = torch.full((4, c["D"]), 0x3C3C, dtype=torch.int16, device="cuda")
    st = tp.tp_mlp_pair(dd["X"], 0, c["D"], c["F"], dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"],
                        c["T"], Y, None, 0)
    assert st == 0
    torch.cuda.synchronize()
    assert np.all(from_dev(Y) == 0x3C3C)
    assert tp.tp_check_device_error() == 0


def test_bench_step_sequence_matches_one_shot(flux):
    # bench.py times the three calls that tp_mlp_pair makes (one batched slice
    # launch, two GEMMs), one by one; they must produce exactly the one-shot result.
    c, d, _ = flux
    M, D, F, T = c["M"], c["D"], c["F"], c["T"]
    Fs = F // T
    dd = _dev(d)
    w_up = torch.empty((T, Fs, D), dtype=torch.int16, device="cuda")
    b_up = torch.empty((T, Fs), dtype=torch.int16, device="cuda")
    w_down = torch.empty((T, D, Fs), dtype=torch.int16, device="cuda")
    H = torch.empty((T, M, Fs), dtype=torch.int16, device="cuda")
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    n0 = tp.tp_kernel_launches()
    jobs = [(dd["W_up"], F, D, tp.TP_COLWISE, w_up), (dd["W_down"], D, F, tp.TP_ROWWISE, w_down),
            (dd["b_up"], T, Fs, tp.TP_COLWISE, b_up)]
    assert tp.tp_shard_weights_batch(jobs, T) == 0
    assert tp.tp_colwise_linear(dd["X"], M, D, w_up, b_up, Fs, T, 1, tp.TP_OUT_BF16, H) == 0
    assert tp.tp_rowwise_linear_sum(H, M, Fs, w_down, D, dd["b_down"], T, Y) == 0
    assert tp.tp_kernel_launches() - n0 == 3
    torch.cuda.synchronize()
    one = _run_pair(dd, M, D, F, T)
    assert np.array_equal(from_dev(Y), one)
    # the stacked shards are the oracle's slices
    for r in (0, T - 1):
        assert np.array_equal(from_dev(w_up[r]), o.slice_colwise(d["W_up"], T, r))
        assert np.array_equal(from_dev(w_down[r]), o.slice_rowwise(d["W_down"], T, r))


def test_bench_step_equals_prepared_run(flux):
    # bench.py's headline step is the two GEMM launches on shards sliced once;
    # they must be exactly what tp_mlp_run does on a tp_mlp_prepare handle.
    c, d, _ = flux
    M, D, F, T = c["M"], c["D"], c["F"], c["T"]
    Fs = F // T
    dd = _dev(d)
    w_up = torch.empty((T, Fs, D), dtype=torch.int16, device="cuda")
    b_up = torch.empty((T, Fs), dtype=torch.int16, device="cuda")
    w_down = torch.empty((T, D, Fs), dtype=torch.int16, device="cuda")
    H = torch.empty((T, M, Fs), dtype=torch.int16, device="cuda")
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    jobs = [(dd["W_up"], F, D, tp.TP_COLWISE, w_up), (dd["W_down"], D, F, tp.TP_ROWWISE, w_down),
            (dd["b_up"], T, Fs, tp.TP_COLWISE, b_up)]
    assert tp.tp_shard_weights_batch(jobs, T) == 0
    n0 = tp.tp_kernel_launches()
    assert tp.tp_colwise_linear(dd["X"], M, D, w_up, b_up, Fs, T, 1, tp.TP_OUT_BF16, H) == 0
    assert tp.tp_rowwise_linear_sum(H, M, Fs, w_down, D, dd["b_down"], T, Y) == 0
    assert tp.tp_kernel_launches() - n0 == 2
    pair = tp.MlpPair(dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T)
    n0 = tp.tp_kernel_launches()
    Yr = pair(dd["X"])
    assert tp.tp_kernel_launches() - n0 == 2
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(Y), from_dev(Yr))
    pair.close()
