"""Attention on the GPU: the per-shard SDPA kernel alone (a6) and the whole
block (a5..a7), against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, assert_rounded_once, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,Hs,T", [(1, 1, 1), (128, 1, 1), (200, 2, 2), (256, 1, 3), (1000, 2, 1), (4608, 1, 1)])
def test_sdpa_step(M, Hs, T):
    W = 3 * Hs * 128
    # Q, K, V of unit variance, like the projections of a unit-variance input (fp16 storage)
    QKV = syn.normal_f16((T, M, W), 1.0, seed=M + Hs, tid=400)
    O = torch.empty((T, M, Hs * 128), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(to_dev(QKV), M, Hs * T, T, O) == 0
    torch.cuda.synchronize()
    g = from_dev(O)
    q = syn.f16_bits_to_f64(QKV)
    for r in range(T):
        for j in range(Hs):
            Q = q[r][:, j * 128:(j + 1) * 128]
            K = q[r][:, (Hs + j) * 128:(Hs + j + 1) * 128]
            V = q[r][:, (2 * Hs + j) * 128:(2 * Hs + j + 1) * 128]
            assert_rounded_once(g[r][:, j * 128:(j + 1) * 128], o.sdpa(Q, K, V), f"sdpa r={r} j={j}")


# More work items (shard, head, 512 query rows) than CTA pairs: the persistent
# kernel walks several items per pair (149 items over 74 pairs; 200 items with
# ragged query and key blocks; 150 items of one whole query block each).
@pytest.mark.parametrize("M,Hs,T", [(256, 149, 1), (333, 100, 2), (512, 150, 1)])
def test_sdpa_several_items_per_cta(M, Hs, T):
    test_sdpa_step(M, Hs, T)


def test_sdpa_large_scores_rescale_path():
    # Scores spread over a wide range force the running-max rescale of O.
    M, Hs, T = 512, 1, 1
    QKV = syn.normal_f16((T, M, 3 * 128), 1.0, seed=7, tid=401)
    q = syn.f16_bits_to_f64(QKV)
    # scale Q up (exact in fp16: a power of two) so that maxima grow along the key sequence
    QKV[0][:, :128] = (q[0][:, :128] * 8.0).astype(np.float16).view(np.uint16)
    q = syn.f16_bits_to_f64(QKV)
    O = torch.empty((T, M, 128), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(to_dev(QKV), M, 1, 1, O) == 0
    torch.cuda.synchronize()
    ref = o.sdpa(q[0][:, :128], q[0][:, 128:256], q[0][:, 256:])
    assert_rounded_once(from_dev(O)[0], ref, "sdpa wide scores")


def test_sdpa_huge_scores():
    # Scores of a few thousand (Q scaled by 64, exact in fp16): the softmax is
    # nearly one-hot and the kernel's row-max estimate sits furthest from the
    # true max; the result must still be the rounded exact attention.
    M = 384
    QKV = syn.normal_f16((1, M, 3 * 128), 1.0, seed=11, tid=402)
    q = syn.f16_bits_to_f64(QKV)
    QKV[0][:, :128] = (q[0][:, :128] * 64.0).astype(np.float16).view(np.uint16)
    q = syn.f16_bits_to_f64(QKV)
    O = torch.empty((1, M, 128), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(to_dev(QKV), M, 1, 1, O) == 0
    torch.cuda.synchronize()
    ref = o.sdpa(q[0][:, :128], q[0][:, 128:256], q[0][:, 256:])
    assert_rounded_once(from_dev(O)[0], ref, "sdpa huge scores")


@pytest.mark.parametrize("M,heads,T", [(200, 4, 2), (64, 2, 1), (333, 4, 4)])
def test_attn_block_small(M, heads, T):
    D = heads * 128
    d = syn.attn_inputs(M, D, seed=M + heads)
    f = {k: f64(v) for k, v in d.items()}
    Y = tp.attn_block(to_dev(d["X"]), to_dev(d["W_qkv"]), to_dev(d["W_o"]), heads, T)
    torch.cuda.synchronize()
    ref = o.attn_sharded_summed(f["X"], f["W_qkv"], f["W_o"], heads, T)
    assert_parity(from_dev(Y), ref, "attn block")


def test_flux_attention_block():
    c = syn.CONFIGS["flux_attn"]
    d = syn.attn_inputs(c["M"], c["D"], c["seed"])
    f = {k: f64(v) for k, v in d.items()}
    dd = {k: to_dev(v) for k, v in d.items()}
    Y = tp.attn_block(dd["X"], dd["W_qkv"], dd["W_o"], c["H"], c["T"])
    torch.cuda.synchronize()
    g = from_dev(Y)
    ref = o.attn_sharded_summed(f["X"], f["W_qkv"], f["W_o"], c["H"], c["T"])
    assert_parity(g, ref, "flux attention")
    layer = tp.AttnBlock(dd["W_qkv"], dd["W_o"], c["H"], c["T"])
    Y2 = layer(dd["X"])
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(Y2), g)
    layer.close()


def test_bench_step_sequence_matches_one_shot():
    # bench.py times the attention block as four step calls (one batched slice
    # launch for W_qkv's head split and W_o, the QKV GEMM, the SDPA, the
    # out-projection); same bits as tp_attn_block.
    import bench
    wl = bench.AttnWorkload(dict(kind="attn", M=384, D=512, H=4, T=2, seed=12))
    d = wl.host_inputs(0)
    g = {k: to_dev(v) for k, v in d.items()}
    n0 = tp.tp_kernel_launches()
    for k in wl.kernels(tp, g, "cuda"):
        k.fn()
    assert tp.tp_kernel_launches() - n0 == 4
    torch.cuda.synchronize()
    Y = tp.attn_block(g["X"], g["W_qkv"], g["W_o"], 4, 2)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(wl.bufs["A"]), from_dev(Y))
