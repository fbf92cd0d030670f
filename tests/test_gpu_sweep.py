"""Seeded sweep of random ragged shapes through the step-level GEMM calls
(both kernels, every epilogue form) against the fp64 oracle: M, K, N drawn so
that tile tails, K-block tails and shard counts vary from case to case."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, assert_rounded_once, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    T = int(rng.choice([1, 2, 3, 4, 8]))
    M = int(rng.integers(1, 700))
    K = 8 * int(rng.integers(1, 60))
    Ns = 8 * int(rng.integers(1, 70))
    return T, M, K, Ns


@pytest.mark.parametrize("seed", range(12))
def test_random_colwise(seed):
    T, M, K, Ns = _case(seed)
    mode = seed % 3  # 0: GELU + bias, 1: plain fp16 out, 2: SwiGLU
    X = syn.normal_bf16((M, K), 1.0, seed=seed, tid=500)
    if mode == 2:
        W = syn.normal_bf16((T, 2 * Ns, K), 1.0 / np.sqrt(K), seed=seed, tid=501)
        b = syn.normal_bf16((T, 2 * Ns), 0.1, seed=seed, tid=502)
        out = torch.zeros((T, M, Ns), dtype=torch.int16, device="cuda")
        assert tp.tp_colwise_swiglu(to_dev(X), M, K, to_dev(W), to_dev(b), Ns, T, out) == 0
        torch.cuda.synchronize()
        g = from_dev(out)
        for r in range(T):
            G = o.linear(f64(X), f64(W[r, :Ns]), f64(b[r, :Ns]))
            U = o.linear(f64(X), f64(W[r, Ns:]), f64(b[r, Ns:]))
            assert_rounded_once(g[r], o.silu(G) * U, f"sweep {seed} swiglu shard {r}")
        return
    W = syn.normal_bf16((T, Ns, K), 1.0 / np.sqrt(K), seed=seed, tid=501)
    b = syn.normal_bf16((T, Ns), 0.1, seed=seed, tid=502) if mode == 0 else None
    out = torch.zeros((T, M, Ns), dtype=torch.int16, device="cuda")
    assert tp.tp_colwise_linear(to_dev(X), M, K, to_dev(W), to_dev(b) if b is not None else None, Ns, T,
                                mode == 0, tp.TP_OUT_F16 if mode == 1 else tp.TP_OUT_BF16, out) == 0
    torch.cuda.synchronize()
    g = from_dev(out)
    for r in range(T):
        ref = o.linear(f64(X), f64(W[r]), f64(b[r]) if b is not None else None)
        if mode == 0:
            assert_rounded_once(g[r], o.gelu_tanh(ref), f"sweep {seed} colwise shard {r}")
        else:
            got = syn.f16_bits_to_f64(g[r])
            rms = np.sqrt(np.mean(ref ** 2))
            assert np.max(np.abs(got - ref)) <= 4e-3 * rms, f"sweep {seed} fp16 shard {r}"


@pytest.mark.parametrize("seed", range(12))
def test_random_rowwise(seed):
    T, M, Ks, N = _case(seed + 100)
    X = syn.normal_bf16((T, M, Ks), 1.0, seed=seed, tid=510)
    W = syn.normal_bf16((T, N, Ks), 1.0 / np.sqrt(T * Ks), seed=seed, tid=511)
    b = syn.normal_bf16((N,), 0.02, seed=seed, tid=512) if seed % 2 else None
    Y = torch.zeros((M, N), dtype=torch.int16, device="cuda")
    if seed % 3 == 2:  # the same sum through rowwise_split_input on the concatenated input
        Xcat = np.concatenate([X[r] for r in range(T)], axis=1)
        assert tp.tp_rowwise_split_input_linear(to_dev(Xcat), M, T * Ks, to_dev(W), N,
                                                to_dev(b) if b is not None else None, T, Y) == 0
    else:
        assert tp.tp_rowwise_linear_sum(to_dev(X), M, Ks, to_dev(W), N, to_dev(b) if b is not None else None, T,
                                        Y) == 0
    torch.cuda.synchronize()
    ref = o.reduce_partials([o.linear(f64(X[r]), f64(W[r])) for r in range(T)], f64(b) if b is not None else None)
    assert_parity(from_dev(Y), ref, f"sweep {seed} rowwise T={T} M={M} Ks={Ks} N={N}")
