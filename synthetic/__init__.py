"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws random numbers and encodes them as bf16 bit patterns.
It holds none of the layer arithmetic (no slicing, no GEMM, no activation,
no softmax), so the oracle and the CUDA path can both consume its output
without sharing any of the method's code.

Generator (one definition, used by everyone):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014).  The stream of tensor ``tid`` under seed ``s``
  starts from ``base = mix(s * GAMMA ^ (tid + 1) * 0xD1B54A32D192ED03)``;
  element ``i`` takes the ``(i + 1)``-th SplitMix64 output of that stream,
  ``r_i = mix(base + (i + 1) * GAMMA)`` (all arithmetic mod 2**64).
* Box-Muller (Box & Muller, 1958): ``u1 = (hi32(r) + 0.5) / 2**32``,
  ``u2 = lo32(r) / 2**32``, ``z = sqrt(-2 ln u1) * cos(2 pi u2)``.
* value = ``float32(z * std)`` (round to nearest even), then bf16 by
  round-to-nearest-even on the float32 bit pattern.

Tensor ids per layer (fixed so that every degree of a sweep sees identical
weights): X=0, W_up=1, b_up=2, W_down=3, b_down=4, W_qkv=5, W_o=6; the MLP of
the composed attention+MLP block uses W_up=7, b_up=8, W_down=9, b_down=10.
Scales: activations std 1, weights std 1/sqrt(fan_in) with fan_in the
input-feature count (dim 1 of an ``[out x in]`` weight), biases std 0.02.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TID_MUL = np.uint64(0xD1B54A32D192ED03)

TID = {
    "X": 0, "W_up": 1, "b_up": 2, "W_down": 3, "b_down": 4,
    "W_qkv": 5, "W_o": 6,
    "W_up2": 7, "b_up2": 8, "W_down2": 9, "b_down2": 10,
    "W_in": 11, "b_in": 12, "W_out": 13, "b_out": 14,
    "X_txt": 15, "W_qkv_txt": 16, "W_o_txt": 17,
}

_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, tid: int) -> np.uint64:
    with np.errstate(over="ignore"):
        a = np.array([seed], dtype=np.uint64) * GAMMA
        b = np.array([tid + 1], dtype=np.uint64) * _TID_MUL
        return _mix(a ^ b)[0]


def _f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = x.astype(np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def _fill(out: np.ndarray, base: np.uint64, std: float, start: int, end: int) -> None:
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, end + 1, dtype=np.uint64)
        r = _mix(base + i * GAMMA)
        u1 = ((r >> np.uint64(32)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
        u2 = (r & np.uint64(0xFFFFFFFF)).astype(np.float64) * (1.0 / 4294967296.0)
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos((2.0 * np.pi) * u2)
        out[start:end] = _f32_to_bf16_bits((z * std).astype(np.float32))


def normal_bf16(shape, std: float, seed: int, tid: int) -> np.ndarray:
    """Seeded N(0, std^2) draws encoded as bf16 bit patterns (uint16 array).

    Element i depends only on (seed, tid, i), so the chunks are filled by a
    thread pool in any order with an identical result.
    """
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.uint16)
    base = _stream_base(seed, tid)
    spans = [(a, min(n, a + _CHUNK)) for a in range(0, n, _CHUNK)]
    if len(spans) <= 1:
        for a, b in spans:
            _fill(out, base, std, a, b)
    else:
        workers = min(len(spans), os.cpu_count() or 1, 32)
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(lambda ab: _fill(out, base, std, ab[0], ab[1]), spans))
    return out.reshape(shape)


def normal_f16(shape, std: float, seed: int, tid: int) -> np.ndarray:
    """The same seeded draws as ``normal_bf16`` (bf16-valued), encoded as fp16 bit
    patterns (uint16).  bf16 values of moderate magnitude are exact in fp16."""
    v = bf16_bits_to_f64(normal_bf16(shape, std, seed, tid))
    return v.astype(np.float16).view(np.uint16)


def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of fp16 bit patterns (uint16) to float64."""
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Encode float64 values as bf16 via float32 (both roundings to nearest even)."""
    return _f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


# ---------------------------------------------------------------------------
# Workloads: one dict of bf16 bit arrays per layer configuration.
# ---------------------------------------------------------------------------

def mlp_inputs(M: int, D: int, F: int, seed: int, ids=("X", "W_up", "b_up", "W_down", "b_down"),
               X: np.ndarray | None = None) -> dict:
    """Inputs of one colwise->rowwise MLP pair: X[M,D], W_up[F,D], b_up[F], W_down[D,F], b_down[D]."""
    x_id, wu_id, bu_id, wd_id, bd_id = (TID[k] for k in ids)
    return {
        "X": normal_bf16((M, D), 1.0, seed, x_id) if X is None else X,
        "W_up": normal_bf16((F, D), 1.0 / np.sqrt(D), seed, wu_id),
        "b_up": normal_bf16((F,), 0.02, seed, bu_id),
        "W_down": normal_bf16((D, F), 1.0 / np.sqrt(F), seed, wd_id),
        "b_down": normal_bf16((D,), 0.02, seed, bd_id),
    }


def attn_inputs(M: int, D: int, seed: int) -> dict:
    """Inputs of one attention block: X[M,D], W_qkv[3D,D] (Q;K;V stacked on dim 0), W_o[D,D]."""
    return {
        "X": normal_bf16((M, D), 1.0, seed, TID["X"]),
        "W_qkv": normal_bf16((3 * D, D), 1.0 / np.sqrt(D), seed, TID["W_qkv"]),
        "W_o": normal_bf16((D, D), 1.0 / np.sqrt(D), seed, TID["W_o"]),
    }


def block_inputs(M: int, D: int, F: int, seed: int) -> dict:
    """Inputs of the composed block: attention (X, W_qkv, W_o) then an MLP pair (ids 7..10)."""
    d = attn_inputs(M, D, seed)
    mlp = mlp_inputs(M, D, F, seed, ids=("X", "W_up2", "b_up2", "W_down2", "b_down2"), X=d["X"])
    d.update({k: mlp[k] for k in ("W_up", "b_up", "W_down", "b_down")})
    return d


def swiglu_inputs(M: int, D: int, F: int, seed: int) -> dict:
    """Inputs of a SwiGLU pair: X[M,D], W_in[2F,D] = [W_gate; W_up], b_in[2F],
    W_out[D,F], b_out[D] (same scales as the GELU pair)."""
    return {
        "X": normal_bf16((M, D), 1.0, seed, TID["X"]),
        "W_in": normal_bf16((2 * F, D), 1.0 / np.sqrt(D), seed, TID["W_in"]),
        "b_in": normal_bf16((2 * F,), 0.02, seed, TID["b_in"]),
        "W_out": normal_bf16((D, F), 1.0 / np.sqrt(F), seed, TID["W_out"]),
        "b_out": normal_bf16((D,), 0.02, seed, TID["b_out"]),
    }


def joint_attn_inputs(M_img: int, M_txt: int, D: int, seed: int) -> dict:
    """Inputs of dual-stream joint attention: the image stream uses the
    attention block's ids (X, W_qkv, W_o), the text stream its own."""
    return {
        "X_img": normal_bf16((M_img, D), 1.0, seed, TID["X"]),
        "X_txt": normal_bf16((M_txt, D), 1.0, seed, TID["X_txt"]),
        "W_qkv_img": normal_bf16((3 * D, D), 1.0 / np.sqrt(D), seed, TID["W_qkv"]),
        "W_qkv_txt": normal_bf16((3 * D, D), 1.0 / np.sqrt(D), seed, TID["W_qkv_txt"]),
        "W_o_img": normal_bf16((D, D), 1.0 / np.sqrt(D), seed, TID["W_o"]),
        "W_o_txt": normal_bf16((D, D), 1.0 / np.sqrt(D), seed, TID["W_o_txt"]),
    }


# The layer configurations exercised by the tests and the benchmark.
CONFIGS = {
    "tiny_mlp": dict(kind="mlp", M=64, D=128, F=512, T=2, seed=0),
    "flux_mlp": dict(kind="mlp", M=4608, D=3072, F=12288, T=4, seed=1),
    "flux_attn": dict(kind="attn", M=4608, D=3072, H=24, T=4, seed=2),
    "flux_mlp_sweep": dict(kind="mlp", M=4608, D=3072, F=12288, T=(1, 2, 4, 8), seed=1),
    "wide_block": dict(kind="block", M=16384, D=6144, H=48, F=24576, T=8, seed=3),
    # SwiGLU pair, gate and up packed with blocks [1, 1], mlp_ratio 3 (F = 3 D)
    "flux_swiglu": dict(kind="swiglu", M=4608, D=3072, F=9216, T=4, seed=4),
    # dual-stream joint attention: 4096 image + 512 text tokens, one SDPA over both
    "flux_joint_attn": dict(kind="joint", M_img=4096, M_txt=512, D=3072, H=24, T=4, seed=6),
}
