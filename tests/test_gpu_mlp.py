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
