"""Context-parallelism pieces on one GPU ("Context parallelism" page, Ring and
Ulysses attention), against the fp64 oracle.

Ring: the per-key-block attention with statistics (tp_sdpa_block_stats) and
the merge of several blocks (tp_attn_merge) must give the attention over all
keys.  Ulysses: packing each rank's Q/K/V by destination head group (packed
rowwise slicing, blocks [1, 1, 1]), the all-to-all (emulated here by moving
blocks between buffers: on several GPUs it is NCCL's), per-rank attention
over all tokens and the regrouping back (tp_unshard_rowwise_all) must give
exactly the single-device attention's bits."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import FROB_REL, MAX_REL_RMS, assert_rounded_once, from_dev, to_dev

pytestmark = pytest.mark.gpu

LN2 = np.log(2.0)


def _heads(q, Hs, j):
    """Q, K, V of head j from a [rows x 3*Hs*128] block of fp64 values."""
    return (q[:, j * 128:(j + 1) * 128], q[:, (Hs + j) * 128:(Hs + j + 1) * 128],
            q[:, (2 * Hs + j) * 128:(2 * Hs + j + 1) * 128])


def _close(got, ref, what):
    rms = np.sqrt(np.mean(ref * ref))
    mx = np.max(np.abs(got - ref)) / rms
    fr = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert mx <= MAX_REL_RMS and fr <= FROB_REL, f"{what}: max/rms={mx:.3e} frob={fr:.3e}"


@pytest.mark.parametrize("Mq,Mk,Hs,T", [(300, 200, 2, 2), (1, 129, 1, 1), (640, 512, 3, 1), (1000, 64, 2, 2)])
def test_block_stats(Mq, Mk, Hs, T):
    cols = 3 * Hs * 128
    Qb = syn.normal_f16((T, Mq, cols), 1.0, seed=Mq, tid=410)
    KVb = syn.normal_f16((T, Mk, cols), 1.0, seed=Mk, tid=411)
    O = torch.empty((T, Mq, Hs * 128), dtype=torch.float16, device="cuda")
    lse = torch.empty((T, Hs, Mq), dtype=torch.float32, device="cuda")
    assert tp.tp_sdpa_block_stats(to_dev(Qb), Mq, to_dev(KVb), Mk, Hs * T, T, O, lse) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    Og, Lg = O.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    q, kv = syn.f16_bits_to_f64(Qb), syn.f16_bits_to_f64(KVb)
    for r in range(T):
        for j in range(Hs):
            Q = _heads(q[r], Hs, j)[0]
            _, K, V = _heads(kv[r], Hs, j)
            ref, ref_lse = o.sdpa(Q, K, V, return_lse=True)
            _close(Og[r][:, j * 128:(j + 1) * 128], ref, f"block O r={r} j={j}")
            assert np.max(np.abs(Lg[r][j] - ref_lse / LN2)) <= 2e-3, "log-sum-exp (log2 units)"


# up to 8 blocks the merge is instantiated per block count; 10 and 12 blocks
# take the run-time-count path
@pytest.mark.parametrize("M,splits,Hs", [(640, [256, 256, 128], 2), (1000, [300, 1, 699], 1), (512, [512], 1),
                                         (640, [64] * 10, 1), (700, [50, 70, 30, 100, 40, 60, 80, 20, 90, 10, 70, 80], 2)])
def test_ring_blocks_merge_to_full_attention(M, splits, Hs):
    # One "rank" holds all M queries; the keys arrive in blocks, as on a ring.
    cols = 3 * Hs * 128
    QKV = syn.normal_f16((1, M, cols), 1.0, seed=M + 1, tid=412)
    full = to_dev(QKV)
    parts_O = torch.empty((len(splits), 1, M, Hs * 128), dtype=torch.float16, device="cuda")
    parts_L = torch.empty((len(splits), 1, Hs, M), dtype=torch.float32, device="cuda")
    j0 = 0
    for b, n in enumerate(splits):
        kv = full[:, j0:j0 + n].contiguous()  # another rank's block of tokens
        assert tp.tp_sdpa_block_stats(full, M, kv, n, Hs, 1, parts_O[b], parts_L[b]) == 0
        j0 += n
    O = torch.empty((1, M, Hs * 128), dtype=torch.int16, device="cuda")
    lse = torch.empty((1, Hs, M), dtype=torch.float32, device="cuda")
    assert tp.tp_attn_merge(parts_O, parts_L, len(splits), M, Hs, 1, O, lse) == 0
    O_ref = torch.empty((1, M, Hs * 128), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(full, M, Hs, 1, O_ref) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    q = syn.f16_bits_to_f64(QKV)[0]
    got = from_dev(O)[0]
    for j in range(Hs):
        Q, K, V = _heads(q, Hs, j)
        ref, ref_lse = o.sdpa(Q, K, V, return_lse=True)
        assert_rounded_once(got[:, j * 128:(j + 1) * 128], ref, f"ring merge head {j}")
        assert np.max(np.abs(lse.cpu().numpy()[0][j] - ref_lse / LN2)) <= 2e-3
    # the merged result agrees with the one-pass kernel to bf16 rounding
    a, b = (np.abs(syn.bf16_bits_to_f64(x)) for x in (got, from_dev(O_ref)[0]))
    assert np.max(np.abs(syn.bf16_bits_to_f64(got) - syn.bf16_bits_to_f64(from_dev(O_ref)[0]))) <= (
        2 ** -7 * np.max(np.maximum(a, b)) + 1e-3)


def test_block_results_near_the_fp16_limit():
    # A block's O is a convex combination of V rows, so V values near the fp16
    # maximum (here up to ~6e4) stay finite in the fp16 block results and in
    # the merge; each block's O is within one fp16 rounding of the oracle's.
    Mq, Mk, Hs = 130, 300, 1
    qkv = syn.f16_bits_to_f64(syn.normal_f16((1, Mk, 3 * 128), 1.0, seed=77, tid=416))
    qkv[:, :, 256:] *= 15000.0  # V: |V| up to ~6e4 (values past 65504 clipped below)
    qkv[:, :, 256:] = np.clip(qkv[:, :, 256:], -65000.0, 65000.0)
    bits = torch.from_numpy(qkv.astype(np.float16)).view(torch.int16).numpy()
    full = to_dev(bits)
    q = syn.f16_bits_to_f64(bits)[0]
    parts_O = torch.empty((2, 1, Mq, 128), dtype=torch.float16, device="cuda")
    parts_L = torch.empty((2, 1, 1, Mq), dtype=torch.float32, device="cuda")
    for b, (j0, n) in enumerate(((0, 170), (170, 130))):
        kv = full[:, j0:j0 + n].contiguous()
        assert tp.tp_sdpa_block_stats(full[:, :Mq].contiguous(), Mq, kv, n, 1, 1, parts_O[b], parts_L[b]) == 0
    O = torch.empty((1, Mq, 128), dtype=torch.int16, device="cuda")
    assert tp.tp_attn_merge(parts_O, parts_L, 2, Mq, 1, 1, O) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    Q = q[:Mq, :128]
    for b, (j0, n) in enumerate(((0, 170), (170, 130))):
        Ob = parts_O[b, 0].float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(Ob)), "fp16 block result overflowed"
        ref = o.sdpa(Q, q[j0:j0 + n, 128:256], q[j0:j0 + n, 256:])
        assert np.max(np.abs(Ob - ref) - 2.0 ** -9 * np.abs(ref)) <= 1e-3 * np.sqrt(np.mean(ref ** 2)), f"block {b}"
    assert_rounded_once(from_dev(O)[0], o.sdpa(Q, q[:, 128:256], q[:, 256:]), "merge near the fp16 limit")


def test_merge_rejects_bad_part_counts():
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    y = torch.zeros(64, dtype=torch.int16, device="cuda")
    assert tp.STATUS[tp.tp_attn_merge(x, x, 0, 1, 1, 1, y)] == "TP_ERR_BAD_SHAPE"
    assert tp.STATUS[tp.tp_attn_merge(x, x, 65, 1, 1, 1, y)] == "TP_ERR_BAD_SHAPE"


@pytest.mark.parametrize("U,H,M", [(2, 4, 512), (4, 8, 600)])
def test_ulysses_regrouping_is_bit_exact_attention(U, H, M):
    cols = 3 * H * 128
    Ms = M // U
    QKV = syn.normal_f16((M, cols), 1.0, seed=U * 100 + H, tid=413)
    full = to_dev(QKV)
    # rank s packs its tokens by destination head group: [U][Ms][3 * (H/U) * 128]
    sends = []
    for s in range(U):
        send = torch.empty((U, Ms, cols // U), dtype=torch.int16, device="cuda")
        assert tp.tp_shard_packed_all(full[s * Ms:(s + 1) * Ms], Ms, cols, tp.TP_ROWWISE, [1, 1, 1], U, send) == 0
        sends.append(send)
    torch.cuda.synchronize()
    # bit-exact layout: the packed block for rank u is the oracle's packed rowwise slice
    for s in (0, U - 1):
        for u in (0, U - 1):
            assert np.array_equal(from_dev(sends[s][u]), o.slice_packed_rowwise(QKV[s * Ms:(s + 1) * Ms],
                                                                                [1, 1, 1], U, u))
    # all-to-all (emulated): rank u receives every rank's block u, in rank (= token) order
    outs = []
    for u in range(U):
        recv = torch.cat([sends[s][u] for s in range(U)]).contiguous()  # [M][3 * (H/U) * 128]
        O_u = torch.empty((M, (H // U) * 128), dtype=torch.int16, device="cuda")
        assert tp.tp_sdpa_shards(recv, M, H // U, 1, O_u) == 0
        outs.append(O_u)
    # reverse all-to-all (emulated) and regroup: rank s gets [U][Ms][(H/U) * 128]
    result = []
    for s in range(U):
        back = torch.stack([outs[u][s * Ms:(s + 1) * Ms] for u in range(U)]).contiguous()
        O_s = torch.empty((Ms, H * 128), dtype=torch.int16, device="cuda")
        assert tp.tp_unshard_rowwise_all(back, Ms, H * 128, U, O_s) == 0
        result.append(O_s)
    got = torch.cat(result)
    ref = torch.empty((M, H * 128), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(full, M, H, 1, ref) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    assert np.array_equal(from_dev(got), from_dev(ref)), "Ulysses regrouping changed bits"
    q = syn.f16_bits_to_f64(QKV)
    j = H - 1
    assert_rounded_once(from_dev(got)[:, j * 128:(j + 1) * 128], o.sdpa(*_heads(q, H, j)), "Ulysses last head")


def test_unshard_inverts_rowwise_slicing():
    rows, cols, T = 37, 96, 4
    W = syn.normal_bf16((rows, cols), 1.0, seed=9, tid=414)
    sh = torch.empty((T, rows, cols // T), dtype=torch.int16, device="cuda")
    back = torch.empty((rows, cols), dtype=torch.int16, device="cuda")
    assert tp.tp_shard_weight_all(to_dev(W), rows, cols, tp.TP_ROWWISE, T, sh) == 0
    assert tp.tp_unshard_rowwise_all(sh, rows, cols, T, back) == 0
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(back), W)


def test_flux_scale_ring_and_ulysses():
    # The flux_attn tokens (4608, 24 heads x 128) over 4 context-parallel ranks,
    # laid out as the bench runs them: Ring steps over all ranks in one launch
    # each (rank r holds block (r - s) mod 4 at step s), the merge, and Ulysses
    # with the ranks as the SDPA's shards.  Sampled rows against the oracle;
    # Ulysses bit-exact against the single-device attention.
    M, H, R = 4608, 24, 4
    D, Ms = H * 128, M // R
    QKV = syn.normal_f16((M, 3 * D), 1.0, seed=46, tid=415)
    full = to_dev(QKV)
    qkv = full.view(R, Ms, 3 * D)
    ring = torch.cat([qkv, qkv]).contiguous()
    blk = Ms * 3 * D
    Ob = torch.empty((R, R, Ms, D), dtype=torch.float16, device="cuda")
    Lb = torch.empty((R, R, H, Ms), dtype=torch.float32, device="cuda")
    for s in range(R):
        kv = ring.data_ptr() + 2 * (R - s) * blk
        assert tp.tp_sdpa_block_stats(qkv, Ms, kv, Ms, H * R, R, Ob[s], Lb[s]) == 0
    Y = torch.empty((R, Ms, D), dtype=torch.int16, device="cuda")
    assert tp.tp_attn_merge(Ob, Lb, R, Ms, H * R, R, Y) == 0
    ref_dev = torch.empty((M, D), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(full, M, H, 1, ref_dev) == 0
    # Ulysses: pack by head group, exchange, attend (ranks = shards), exchange back, unpack
    send = torch.empty((R, R, Ms, 3 * D // R), dtype=torch.int16, device="cuda")
    jobs = [(qkv[s], Ms, 3 * D, tp.TP_ROWWISE, send[s], [1, 1, 1]) for s in range(R)]
    assert tp.tp_shard_weights_batch(jobs, R) == 0
    recv = send.transpose(0, 1).contiguous()
    O = torch.empty((R, M, D // R), dtype=torch.int16, device="cuda")
    assert tp.tp_sdpa_shards(recv, M, H, R, O) == 0
    back = O.view(R, R, Ms, D // R).transpose(0, 1).contiguous()
    Yu = torch.empty((R, Ms, D), dtype=torch.int16, device="cuda")
    for s in range(R):
        assert tp.tp_unshard_rowwise_all(back[s], Ms, D, R, Yu[s]) == 0
    torch.cuda.synchronize()
    assert tp.tp_check_device_error() == 0
    assert np.array_equal(from_dev(Yu).reshape(M, D), from_dev(ref_dev)), "Ulysses regrouping changed bits"
    rng = np.random.default_rng(46)
    rows = np.unique(np.r_[0, M - 1, rng.choice(M, 30, replace=False)])
    q = syn.f16_bits_to_f64(QKV)
    got = from_dev(Y).reshape(M, D)
    for j in (0, H - 1):
        Qj, Kj, Vj = _heads(q, H, j)
        ref = o.sdpa(Qj[rows], Kj, Vj)
        assert_rounded_once(got[rows, j * 128:(j + 1) * 128], ref, f"flux Ring head {j}")
