"""Error paths on the GPU: a rejected call returns its status and writes
nothing (canary-filled outputs stay intact); the library keeps working after."""
import numpy as np
import pytest
import torch

import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import from_dev, to_dev

pytestmark = pytest.mark.gpu

CANARY = 0x7B7B
S = {v: k for k, v in tp.STATUS.items()}


def test_rejected_calls_write_nothing():
    M, D, F = 64, 128, 512
    d = {k: to_dev(v) for k, v in syn.mlp_inputs(M, D, F, 0).items()}
    Y = torch.full((M, D), CANARY, dtype=torch.int16, device="cuda")
    ws = torch.full((tp.tp_mlp_workspace_bytes(M, D, F, 2),), 0x11, dtype=torch.uint8, device="cuda")
    nb = ws.numel()
    cases = [
        (dict(T=3), "TP_ERR_INDIVISIBLE"),
        (dict(T=0), "TP_ERR_BAD_DEGREE"),
        (dict(nb=100), "TP_ERR_WORKSPACE"),
        (dict(X=None), "TP_ERR_NULL"),
    ]
    for over, want in cases:
        a = dict(X=d["X"], T=2, nb=nb)
        a.update(over)
        st = tp.tp_mlp_pair(a["X"], M, D, F, d["W_up"], d["b_up"], d["W_down"], d["b_down"], a["T"], Y, ws,
                            a["nb"])
        assert st == S[want]
    torch.cuda.synchronize()
    assert np.all(from_dev(Y) == CANARY)
    assert bool((ws == 0x11).all())
    # heads not divisible by the degree
    Xa = to_dev(syn.normal_bf16((M, 768), 1.0, 1, 0))
    Wq = torch.zeros((3 * 768, 768), dtype=torch.int16, device="cuda")
    Wo = torch.zeros((768, 768), dtype=torch.int16, device="cuda")
    Ya = torch.full((M, 768), CANARY, dtype=torch.int16, device="cuda")
    wsa = torch.empty((tp.tp_attn_workspace_bytes(M, 768, 6, 2),), dtype=torch.uint8, device="cuda")
    assert tp.tp_attn_block(Xa, M, 768, Wq, Wo, 6, 4, Ya, wsa, wsa.numel()) == S["TP_ERR_HEADS_INDIVISIBLE"]
    torch.cuda.synchronize()
    assert np.all(from_dev(Ya) == CANARY)
    # and a valid call afterwards succeeds
    assert tp.tp_mlp_pair(d["X"], M, D, F, d["W_up"], d["b_up"], d["W_down"], d["b_down"], 2, Y, ws, nb) == 0
    assert tp.tp_check_device_error() == 0
    assert not np.all(from_dev(Y) == CANARY)


def test_bounded_wait_reports_timeout_and_context_survives():
    # A wait on an mbarrier that nothing arrives on must give up after its limit,
    # leave TP_ERR_DEVICE_TIMEOUT for the host and keep the context usable.
    import time
    assert tp.tp_check_device_error() == 0
    t0 = time.perf_counter()
    assert tp.tp_debug_watchdog(50) == 0
    st = tp.tp_check_device_error()
    dt = time.perf_counter() - t0
    assert tp.STATUS[st] == "TP_ERR_DEVICE_TIMEOUT"
    assert 0.04 < dt < 30.0
    assert tp.tp_check_device_error() == 0  # the error word was cleared
    # the library still works afterwards
    M, D, F = 64, 128, 512
    d = {k: to_dev(v) for k, v in syn.mlp_inputs(M, D, F, 0).items()}
    Y = tp.mlp_pair(d["X"], d["W_up"], d["b_up"], d["W_down"], d["b_down"], 2)
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    assert np.all(np.isfinite(syn.bf16_bits_to_f64(from_dev(Y))))
    assert tp.tp_debug_watchdog(0) == S["TP_ERR_BAD_SHAPE"]
