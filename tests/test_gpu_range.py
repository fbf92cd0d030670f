"""fp16 range of the attention path's Q/K/V: a projection value outside the
fp16 range must be reported (TP_ERR_RANGE from tp_check_device_error), not
passed on as silent infinities, and the context must stay usable.

The inputs are ordinary numbers built on the host: a single product
X[i, k] * W[j, k] lands just inside (65280) or just outside (65536) the fp16
range, whose largest finite value is 65504 (values from 65520 up round to
+inf).  No fault is involved."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu

BF16_ONE = 0x3F80
BF16_65280 = 0x477F  # largest bf16 below 65504: finite in fp16 (0x7BF8)
BF16_65536 = 0x4780  # 2^16: rounds to fp16 +inf


def _colwise_f16(w_bits):
    """One nonzero product at shard 1, row 299, column 199 (the ragged corner of
    a multi-tile problem); returns (status of the device check, output bits)."""
    M, K, Ns, T = 300, 64, 200, 2
    X = np.zeros((M, K), dtype=np.uint16)
    X[299, 5] = BF16_ONE
    W = np.zeros((T, Ns, K), dtype=np.uint16)
    W[1, 199, 5] = w_bits
    out = torch.zeros((T, M, Ns), dtype=torch.int16, device="cuda")
    assert tp.tp_check_device_error() == 0
    assert tp.tp_colwise_linear(to_dev(X), M, K, to_dev(W), None, Ns, T, 0, tp.TP_OUT_F16, out) == 0
    st = tp.tp_check_device_error()
    return st, from_dev(out)


def test_fp16_output_just_inside_the_range_is_not_flagged():
    st, out = _colwise_f16(BF16_65280)
    assert tp.STATUS[st] == "TP_OK"
    assert out[1, 299, 199] == 0x7BF8  # 65280 = 2^15 * (1 + 1016/1024) in fp16
    out[1, 299, 199] = 0
    assert not out.any()


def test_fp16_output_outside_the_range_is_reported():
    st, out = _colwise_f16(BF16_65536)
    assert tp.STATUS[st] == "TP_ERR_RANGE"
    assert out[1, 299, 199] == 0x7C00  # +inf: the value is still written, the status says so
    assert tp.tp_check_device_error() == 0  # reported once, then cleared


def test_attention_block_reports_overflowing_q_and_recovers():
    M, heads, T = 256, 2, 2
    D = heads * 128
    a = syn.attn_inputs(M, D, seed=41)
    X, W_qkv = a["X"].copy(), a["W_qkv"].copy()
    X[7, :] = 0x4100  # 8.0
    W_qkv[3, :] = 0x4280  # 64.0: Q[7, 3] = 256 * 8 * 64 = 131072 > 65504
    Y = tp.attn_block(to_dev(X), to_dev(W_qkv), to_dev(a["W_o"]), heads, T)
    torch.cuda.synchronize()
    assert tp.STATUS[tp.tp_check_device_error()] == "TP_ERR_RANGE"
    del Y
    # the same layer on in-range inputs afterwards: no flag, oracle parity
    fa = {k: f64(v) for k, v in a.items()}
    Y = tp.attn_block(to_dev(a["X"]), to_dev(a["W_qkv"]), to_dev(a["W_o"]), heads, T)
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    assert_parity(from_dev(Y), o.attn_sharded_summed(fa["X"], fa["W_qkv"], fa["W_o"], heads, T),
                  "attention block after a range error")


def test_in_range_flux_attention_projection_sets_no_flag():
    # The flux-scale QKV projection (unit-variance activations) stays far inside fp16.
    c = syn.CONFIGS["flux_attn"]
    M, D, H, T = c["M"], c["D"], c["H"], c["T"]
    a = syn.attn_inputs(M, D, c["seed"])
    Y = tp.attn_block(to_dev(a["X"]), to_dev(a["W_qkv"]), to_dev(a["W_o"]), H, T)
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    assert np.all(np.isfinite(f64(from_dev(Y))))
