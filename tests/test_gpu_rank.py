"""One rank's share of a layer under tensor parallelism across processes
(tp_mlp_rank_partial, tp_attn_rank_partial), on one GPU: the T ranks'
partials are computed one after another from each rank's own shards, then
summed with the standalone reduction (tp_reduce_partials, the per-element
meaning of the AllReduce) with the rowwise bias added once.  The result must
match the fp64 oracle's unsharded layer within the parity tolerance, and
each rank's fp32 partial must match the oracle's partial of that rank.  The
NCCL wiring of the same objects (one rank, a real process group) is checked
last."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tensor_transformer_layers_b200.dist import AttnRank, MlpRank
from tests._util import FROB_REL, MAX_REL_RMS, assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _close_f32(got, ref, what):
    got = got.astype(np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    mx = np.max(np.abs(got - ref)) / rms
    fr = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    print(f"[parity] {what}: max|d|/rms={mx:.3e} frob={fr:.3e}")
    assert mx <= MAX_REL_RMS and fr <= FROB_REL, f"{what}: max/rms={mx:.3e} frob={fr:.3e}"


def _rows(M):
    return np.arange(M) if M <= 512 else np.unique(np.r_[0, M - 1, np.arange(0, M, 97)])


@pytest.mark.parametrize("name", ["tiny_mlp", "flux_mlp"])
def test_mlp_rank_partials_sum_to_the_layer(name):
    c = syn.CONFIGS[name]
    M, D, F, T = c["M"], c["D"], c["F"], c["T"]
    d = syn.mlp_inputs(M, D, F, c["seed"])
    dd = {k: to_dev(v) for k, v in d.items()}
    parts = torch.empty((T, M, D), dtype=torch.float32, device="cuda")
    for r in range(T):
        MlpRank(dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], T, r).partial(dd["X"], out=parts[r])
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    assert tp.tp_reduce_partials(parts, M, D, T, dd["b_down"], Y) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    rows = _rows(M)
    f = {k: f64(v) for k, v in d.items()}
    X = f["X"][rows]
    assert_parity(from_dev(Y)[rows], o.mlp_unsharded(X, f["W_up"], f["b_up"], f["W_down"], f["b_down"]),
                  f"{name}: sum of rank partials")
    P = parts.cpu().numpy()
    for r in (0, T - 1):
        want = o.mlp_rowwise_partial(o.mlp_colwise_shard(X, f["W_up"], f["b_up"], T, r), f["W_down"], T, r)
        _close_f32(P[r][rows], want, f"{name}: rank {r} partial")


def test_attn_rank_partials_sum_to_the_layer():
    M, heads, T = 300, 4, 2
    D = heads * 128
    a = syn.attn_inputs(M, D, seed=12)
    da = {k: to_dev(v) for k, v in a.items()}
    parts = torch.empty((T, M, D), dtype=torch.float32, device="cuda")
    for r in range(T):
        AttnRank(da["W_qkv"], da["W_o"], heads, T, r).partial(da["X"], out=parts[r])
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    assert tp.tp_reduce_partials(parts, M, D, T, None, Y) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    f = {k: f64(v) for k, v in a.items()}
    assert_parity(from_dev(Y), o.attn_unsharded(f["X"], f["W_qkv"], f["W_o"], heads), "attention rank partials")


def test_flux_attention_rank_partials():
    c = syn.CONFIGS["flux_attn"]
    M, D, H, T = c["M"], c["D"], c["H"], c["T"]
    a = syn.attn_inputs(M, D, c["seed"])
    da = {k: to_dev(v) for k, v in a.items()}
    parts = torch.empty((T, M, D), dtype=torch.float32, device="cuda")
    for r in range(T):
        AttnRank(da["W_qkv"], da["W_o"], H, T, r).partial(da["X"], out=parts[r])
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    assert tp.tp_reduce_partials(parts, M, D, T, None, Y) == 0
    torch.cuda.synchronize()
    rows = _rows(M)
    f = {k: f64(v) for k, v in a.items()}
    assert_parity(from_dev(Y)[rows], o.attn_rows(f["X"], f["W_qkv"], f["W_o"], H, rows, tp_degree=T),
                  "flux attention rank partials")


def test_rank_forward_through_a_process_group():
    # One rank, a real NCCL process group: partial -> all_reduce -> bias once.
    import datetime

    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        c = syn.CONFIGS["tiny_mlp"]
        M, D, F = c["M"], c["D"], c["F"]
        d = syn.mlp_inputs(M, D, F, c["seed"])
        dd = {k: to_dev(v) for k, v in d.items()}
        Y = MlpRank(dd["W_up"], dd["b_up"], dd["W_down"], dd["b_down"], 1, 0).forward(dd["X"])
        torch.cuda.synchronize()
        f = {k: f64(v) for k, v in d.items()}
        assert_parity(from_dev(Y), o.mlp_unsharded(f["X"], f["W_up"], f["b_up"], f["W_down"], f["b_down"]),
                      "one-rank group forward")
    finally:
        dist.destroy_process_group()
