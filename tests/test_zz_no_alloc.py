"""The allocation-free MLP pair (tp_mlp_pair_sharded_noalloc), through the C ABI.

It exists for callers that must not allocate device memory (memory owned by
another allocator, or no tolerance for the synchronisation of cudaMalloc /
cudaFree); its hidden activations live in a fixed 64 MiB library array.  Two
calls in a row, on different tokens, must each match the fp64 oracle and the
one-shot tp_mlp_pair on the same inputs within the parity tolerance: the
second call runs on the scratch the first one left behind.  The flux-scale
cases need two row chunks of 2688 tokens at most (the second one ragged in
the 4608 + 77 case).  This file is collected last so that a failure here comes
after every other test ran."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu

CANARY = 0x7B7B
CHUNK = 2688  # rows per chunk at F = 12288: floor(64 MiB / (2 F)) rounded down to a multiple of 128


def _sample_rows(M, seed):
    """Every row of a small case; else rows 0 and M-1, both sides of every
    chunk boundary and one seeded row in every 128-row GEMM tile."""
    if M <= 512:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    rows = [0, M - 1] + [r for b in range(CHUNK, M, CHUNK) for r in (b - 1, b, b + 1) if r < M]
    rows += [t + int(rng.integers(0, min(128, M - t))) for t in range(0, M, 128)]
    return np.unique(np.array(rows))


def _shards(dd, D, F, T, with_bias):
    """What each rank holds after sharded loading, produced without the library allocating."""
    Fs = F // T
    w_up = torch.empty((T, Fs, D), dtype=torch.int16, device="cuda")
    w_down = torch.empty((T, D, Fs), dtype=torch.int16, device="cuda")
    assert tp.tp_shard_weight_all(dd["W_up"], F, D, tp.TP_COLWISE, T, w_up) == 0
    assert tp.tp_shard_weight_all(dd["W_down"], D, F, tp.TP_ROWWISE, T, w_down) == 0
    b_up = None
    if with_bias:
        b_up = torch.empty((T, Fs), dtype=torch.int16, device="cuda")
        assert tp.tp_shard_weight_all(dd["b_up"], T, Fs, tp.TP_COLWISE, T, b_up) == 0
    return w_up, b_up, w_down


@pytest.mark.parametrize("name,M,with_bias", [("tiny_mlp", 64, True), ("tiny_mlp", 200, False),
                                              ("flux_mlp", 4608, True), ("flux_mlp", CHUNK + 77, True)])
def test_noalloc_matches_oracle_and_one_shot_on_two_calls_in_a_row(name, M, with_bias):
    c = syn.CONFIGS[name]
    D, F, T = c["D"], c["F"], c["T"]
    d = syn.mlp_inputs(M, D, F, c["seed"])
    if not with_bias:
        d["b_up"] = d["b_down"] = None
    dd = {k: (None if v is None else to_dev(v)) for k, v in d.items()}
    Xb_bits = syn.normal_bf16((M, D), 1.0, seed=c["seed"] + 77, tid=0)
    w_up, b_up, w_down = _shards(dd, D, F, T, with_bias)
    rows = _sample_rows(M, c["seed"])
    fw = {k: (None if d[k] is None else f64(d[k])) for k in ("W_up", "b_up", "W_down", "b_down")}
    for X_bits, what in ((d["X"], "first call"), (Xb_bits, "second call")):
        X = to_dev(X_bits)
        ws = torch.empty(tp.tp_mlp_workspace_bytes(M, D, F, T), dtype=torch.uint8, device="cuda")
        ref_dev = torch.empty((M, D), dtype=torch.int16, device="cuda")
        assert tp.tp_mlp_pair(X, M, D, F, dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T, ref_dev, ws,
                              ws.numel()) == 0
        Y = torch.full((M, D), CANARY, dtype=torch.int16, device="cuda")
        st = tp.tp_mlp_pair_sharded_noalloc(X, M, D, F, w_up, b_up, w_down, dd["b_down"], T, Y)
        assert st == 0, tp.tp_status_string(st)
        torch.cuda.synchronize()
        got = from_dev(Y)
        ref_oracle = o.mlp_sharded_summed(f64(X_bits[rows]), fw["W_up"], fw["b_up"], fw["W_down"], fw["b_down"], T)
        assert_parity(got[rows], ref_oracle, f"{name} M={M} {what} vs oracle")
        assert_parity(got, f64(from_dev(ref_dev)), f"{name} M={M} {what} vs tp_mlp_pair")
    assert tp.tp_check_device_error() == 0


def test_noalloc_changes_no_free_device_memory_after_its_first_call():
    # The first call on a device may make the driver create the 64 MiB array
    # (lazy module loading); from then on a call allocates nothing.
    c = syn.CONFIGS["tiny_mlp"]
    M, D, F, T = 300, c["D"], c["F"], c["T"]
    d = {k: to_dev(v) for k, v in syn.mlp_inputs(M, D, F, c["seed"]).items()}
    w_up, b_up, w_down = _shards(d, D, F, T, True)
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    assert tp.tp_mlp_pair_sharded_noalloc(d["X"], M, D, F, w_up, b_up, w_down, d["b_down"], T, Y) == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert tp.tp_mlp_pair_sharded_noalloc(d["X"], M, D, F, w_up, b_up, w_down, d["b_down"], T, Y) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
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
