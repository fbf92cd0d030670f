"""Colwise (a2/a3/a5) and rowwise (a4/a7) tcgen05 GEMMs against the oracle,
including ragged M, N and K tails and tiny sizes, on each of the three
tilings (CTA pairs 256x256, one CTA 128x256, one CTA 128x128)."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, assert_rounded_once, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


PAIR, CTA256, CTA128 = 0, 1, 2  # tp_gemm_tile_plan codes

COLWISE = [
    (64, 128, 256, 2, True, True, False),     # tiny MLP's FFN-in
    (1, 64, 8, 1, False, False, False),
    (129, 72, 264, 3, True, True, False),     # ragged M, N and K tails
    (300, 1024, 512, 4, False, True, False),
    (256, 3072, 2304, 1, False, False, True),  # one QKV shard of the Flux attention block (fp16 out)
    (129, 72, 264, 3, True, True, True),
    (257, 72, 264, 3, True, True, False),     # one row into a second 256-row block
    (512, 192, 520, 2, False, True, False),   # ragged N
    (200, 72, 2568, 4, True, True, False),    # 128x256 tiles: 128x128 tiles would take two rounds
    (200, 72, 2568, 4, False, False, True),
    (1025, 72, 2056, 4, True, True, False),   # CTA pairs, ragged M and N, three rounds of tiles
    (1025, 72, 2056, 4, False, True, True),
]


def test_colwise_cases_cover_every_tiling():
    plans = {tp.tp_gemm_tile_plan(M, Ns, T) for (M, K, Ns, T, *_) in COLWISE}
    assert plans == {PAIR, CTA256, CTA128}
    assert tp.tp_gemm_tile_plan(200, 2568, 4) == CTA256
    assert tp.tp_gemm_tile_plan(1025, 2056, 4) == PAIR
    assert tp.tp_gemm_tile_plan(512, 520, 2) == CTA128


@pytest.mark.parametrize("M,K,Ns,T,gelu,bias,f16", COLWISE)
def test_colwise(M, K, Ns, T, gelu, bias, f16):
    X = syn.normal_bf16((M, K), 1.0, seed=M, tid=300)
    W = syn.normal_bf16((T, Ns, K), 1.0 / np.sqrt(K), seed=K, tid=301)
    b = syn.normal_bf16((T, Ns), 0.02, seed=Ns, tid=302) if bias else None
    out = torch.empty((T, M, Ns), dtype=torch.int16, device="cuda")
    st = tp.tp_colwise_linear(to_dev(X), M, K, to_dev(W), to_dev(b) if bias else None, Ns, T, gelu,
                              tp.TP_OUT_F16 if f16 else tp.TP_OUT_BF16, out)
    assert st == 0
    torch.cuda.synchronize()
    g = from_dev(out)
    act = o.gelu_tanh if gelu else (lambda x: x)
    for r in range(T):
        ref = act(o.linear(f64(X), f64(W[r]), f64(b[r]) if bias else None))
        if f16:
            # fp16 keeps 3 more significand bits than bf16: a tighter bound applies
            got = syn.f16_bits_to_f64(g[r])
            rms = np.sqrt(np.mean(ref ** 2))
            assert np.max(np.abs(got - ref)) <= 4e-3 * rms
            assert np.linalg.norm(got - ref) <= 1e-3 * np.linalg.norm(ref)
        else:
            # H_r is an intermediate rounded once to bf16 (GELU outputs are skewed:
            # many near-zero values, a long positive tail)
            assert_rounded_once(g[r], ref, f"colwise shard {r}")


ROWWISE = [
    (64, 256, 128, 2, True),           # tiny MLP's FFN-out
    (1, 8, 8, 1, True),
    (129, 72, 264, 3, True),           # ragged
    (300, 512, 520, 4, False),
    (256, 768, 3072, 4, False),        # Flux attention out-projection shards
    (257, 72, 264, 3, True),           # ragged everywhere
    (1024, 1536, 520, 8, True),        # 8 shards in one K loop
    (512, 768, 3072, 4, True),         # a 512-token text stream's out-projection: 128x128 tiles
    (232, 72, 20488, 2, True),         # 128x256 tiles, ragged N
    (2305, 72, 2056, 8, True),         # CTA pairs, ragged M and N, 8 shards in one K loop
]


def test_rowwise_cases_cover_every_tiling():
    plans = {tp.tp_gemm_tile_plan(M, N, 1) for (M, Ks, N, T, _) in ROWWISE}
    assert plans == {PAIR, CTA256, CTA128}
    assert tp.tp_gemm_tile_plan(512, 3072, 1) == CTA128
    assert tp.tp_gemm_tile_plan(2305, 2056, 1) == PAIR


def test_swiglu_never_takes_128_column_tiles():
    for M in (1, 64, 200, 256, 512, 4096):
        assert tp.tp_gemm_tile_plan(M, 1024, 1, swiglu=True) == (PAIR if M >= 256 else CTA256)


@pytest.mark.parametrize("M,Ks,N,T,bias", ROWWISE)
def test_rowwise_sum(M, Ks, N, T, bias):
    A = syn.normal_bf16((T, M, Ks), 1.0, seed=M, tid=310)
    W = syn.normal_bf16((T, N, Ks), 1.0 / np.sqrt(T * Ks), seed=Ks, tid=311)
    b = syn.normal_bf16((N,), 0.02, seed=N, tid=312) if bias else None
    Y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    st = tp.tp_rowwise_linear_sum(to_dev(A), M, Ks, to_dev(W), N, to_dev(b) if bias else None, T, Y)
    assert st == 0
    torch.cuda.synchronize()
    ref = o.reduce_partials([o.linear(f64(A[r]), f64(W[r])) for r in range(T)], f64(b) if bias else None)
    assert_parity(from_dev(Y), ref, "rowwise")


def test_colwise_identity_weight_passes_input_through():
    # W = I (bf16 exact) and no bias: every output equals its input exactly.
    M, K = 200, 256
    X = syn.normal_bf16((M, K), 1.0, seed=5, tid=320)
    I = syn.f64_to_bf16_bits(np.eye(K))
    out = torch.empty((1, M, K), dtype=torch.int16, device="cuda")
    assert tp.tp_colwise_linear(to_dev(X), M, K, to_dev(I), None, K, 1, 0, tp.TP_OUT_BF16, out) == 0
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(out)[0], X)
