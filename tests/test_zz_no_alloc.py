"""The allocation-free MLP pair (tp_mlp_pair_sharded_noalloc), through the C ABI.

It exists for callers that must not allocate device memory (memory owned by
another allocator, or no tolerance for the synchronisation of cudaMalloc /
cudaFree); its hidden activations live in a fixed 64 MiB library array.  Two
calls in a row, on different tokens, must each match tp_mlp_pair on the same
inputs within the parity tolerance: the second call runs on the scratch the
first one left behind.  The flux-scale case needs two row chunks.  This file
is collected last so that a failure here comes after every other test ran."""
import numpy as np
import pytest
import torch

import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import FROB_REL, MAX_REL_RMS, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu

CANARY = 0x7B7B


def _close(g_bits, ref_bits, what):
    g, ref = f64(g_bits), f64(ref_bits)
    rms = np.sqrt(np.mean(ref * ref))
    max_rel = np.max(np.abs(g - ref)) / rms
    frob = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert max_rel <= MAX_REL_RMS and frob <= FROB_REL, f"{what}: max/rms={max_rel:.3e} frob={frob:.3e}"


@pytest.mark.parametrize("name", ["tiny_mlp", "flux_mlp"])
def test_noalloc_matches_one_shot_on_two_calls_in_a_row(name):
    c = syn.CONFIGS[name]
    M, D, F, T = c["M"], c["D"], c["F"], c["T"]
    Fs = F // T
    d = syn.mlp_inputs(M, D, F, c["seed"])
    dd = {k: to_dev(v) for k, v in d.items()}
    Xb = to_dev(syn.normal_bf16((M, D), 1.0, seed=c["seed"] + 77, tid=0))
    # what each rank holds after sharded loading, produced without allocating in the library
    w_up = torch.empty((T, Fs, D), dtype=torch.int16, device="cuda")
    b_up = torch.empty((T, Fs), dtype=torch.int16, device="cuda")
    w_down = torch.empty((T, D, Fs), dtype=torch.int16, device="cuda")
    assert tp.tp_shard_weight_all(dd["W_up"], F, D, tp.TP_COLWISE, T, w_up) == 0
    assert tp.tp_shard_weight_all(dd["b_up"], T, Fs, tp.TP_COLWISE, T, b_up) == 0
    assert tp.tp_shard_weight_all(dd["W_down"], D, F, tp.TP_ROWWISE, T, w_down) == 0
    ref_a = from_dev(tp.mlp_pair(dd["X"], dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T))
    ref_b = from_dev(tp.mlp_pair(Xb, dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T))
    for X, ref, what in ((dd["X"], ref_a, "first call"), (Xb, ref_b, "second call")):
        Y = torch.full((M, D), CANARY, dtype=torch.int16, device="cuda")
        st = tp.tp_mlp_pair_sharded_noalloc(X, M, D, F, w_up, b_up, w_down, dd["b_down"], T, Y)
        assert st == 0, tp.tp_status_string(st)
        torch.cuda.synchronize()
        _close(from_dev(Y), ref, f"{name} {what}")
    assert tp.tp_check_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # F = 262152: 128 rows of hidden activations need 2*F*128 bytes > 64 MiB.
    D, F, M = 8, 262152, 4
    X = torch.zeros((M, D), dtype=torch.int16, device="cuda")
    Y = torch.full((M, D), CANARY, dtype=torch.int16, device="cuda")
    fake = 1 << 20  # never dereferenced: the size check fails before anything is launched
    st = tp.tp_mlp_pair_sharded_noalloc(X, M, D, F, fake, None, fake, None, 1, Y)
    assert tp.STATUS[st] == "TP_ERR_SCRATCH_LIMIT"
    assert "64 MiB" in tp.tp_status_string(st)
    torch.cuda.synchronize()
    assert np.all(from_dev(Y) == CANARY)
