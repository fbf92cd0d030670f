"""fp64 CPU oracle for the tensor-parallel (TP) layer pair.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (``tensor_transformer_layers_b200``); the two meet only in
the seeded input generator ``synthetic``.

The arithmetic is plain C++17 in fp64 (``oracle.cpp``, OpenMP over output
rows, built into ``liboracle.so`` by ``oracle/build.py``); this module only
marshals numpy arrays to it and turns its status codes into ValueError.
What each function computes, and the passage it follows (Diffusers
documentation, "Tensor parallelism" page, Portuguese "main" and Chinese
v0.43.0 editions; "Context parallelism" page for the Ring / Ulysses pieces),
is stated in ``oracle.cpp`` beside the code and summarised here:

* style table ("Colwise and rowwise"): colwise slices weight dim 0, rowwise
  weight dim 1; the paragraph under it: a colwise -> rowwise pair needs one
  AllReduce (sum of the rowwise partials), colwise Q/K/V split the heads;
* "Fused projections": packed Linears are sliced block by block;
* "Constraints and validation": the degree divides the heads and every packed
  block (checked before any slicing), and the sharded output equals the
  single-device output -- the definition every layer below is written from.

Readings where the pages are silent: tanh-form GELU (Hendrycks & Gimpel
2016); SiLU x / (1 + e^-x) (Elfwing et al. 2018) for SwiGLU = silu(gate) * up
with W_in = [W_gate; W_up]; the rowwise bias added once after the sum; fused
QKV = [Q; K; V] on dim 0 with head h at rows h*128.. of each block; attention
softmax(Q K^T / sqrt(128)) V per head, non-causal, two-pass softmax; the
composed block mlp_pair(attn_block(X)) with a bf16 hand-off between layers;
sums over shards in ascending shard order.
"""
from __future__ import annotations

import contextlib
import ctypes

import numpy as np

from . import build as _build

HEAD_DIM = 128

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double

_SIGS = {
    "oracle_num_threads": [],
    "oracle_slice_colwise": [_P, _I64, _I64, _I64, _I, _I, _P],
    "oracle_slice_rowwise": [_P, _I64, _I64, _I64, _I, _I, _P],
    "oracle_packed_block_sizes": [_I64, _P, _I, _I, _P],
    "oracle_slice_packed_colwise": [_P, _I64, _I64, _I64, _P, _I, _I, _I, _P],
    "oracle_slice_packed_rowwise": [_P, _I64, _I64, _I64, _P, _I, _I, _I, _P],
    "oracle_slice_qkv_heads": [_P, _I64, _I64, _I64, _I, _I, _I, _P],
    "oracle_check_heads": [_I64, _I, _I],
    "oracle_linear": [_P, _I64, _I64, _P, _I64, _P, _P],
    "oracle_gelu_tanh": [_P, _I64, _P],
    "oracle_silu": [_P, _I64, _P],
    "oracle_softmax_rows": [_P, _I64, _I64, _P],
    "oracle_sdpa": [_P, _I64, _P, _P, _I64, _I64, _D, _P, _P],
    "oracle_reduce_partials": [_P, _I, _I64, _I64, _P, _P],
    "oracle_attn_merge": [_P, _P, _I, _I64, _I64, _P, _P],
    "oracle_mlp_colwise_shard": [_P, _I64, _I64, _P, _P, _I64, _I, _I, _I, _P],
    "oracle_mlp_rowwise_partial": [_P, _I64, _P, _I64, _I64, _I, _I, _P],
    "oracle_mlp_sharded_summed": [_P, _I64, _I64, _P, _P, _I64, _P, _P, _I, _I, _P],
    "oracle_mlp_unsharded": [_P, _I64, _I64, _P, _P, _I64, _P, _P, _I, _P],
    "oracle_swiglu_unsharded": [_P, _I64, _I64, _P, _P, _I64, _P, _P, _P],
    "oracle_swiglu_sharded_summed": [_P, _I64, _I64, _P, _P, _I64, _P, _P, _I, _P],
    "oracle_rowwise_split_input": [_P, _I64, _I64, _P, _I64, _P, _I, _P],
    "oracle_attn_unsharded": [_P, _I64, _I64, _P, _P, _I, _P],
    "oracle_attn_shard_output": [_P, _I64, _I64, _P, _I, _I, _I, _P],
    "oracle_attn_rows": [_P, _I64, _I64, _P, _P, _I, _P, _I64, _I, _P],
    "oracle_joint_attn_unsharded": [_P, _I64, _P, _I64, _I64, _P, _P, _P, _P, _I, _P, _P],
    "oracle_joint_attn_rows": [_P, _I64, _P, _I64, _I64, _P, _P, _P, _P, _I, _P, _I64, _P, _I64, _I, _P, _P],
}

_ERRORS = {
    -1: "tp_degree must be >= 1",
    -2: "rank outside [0, tp_degree)",
    -3: "a sharded dimension (or packed block) is not divisible by tp_degree",
    -4: "tp_degree does not divide the number of heads",
    -5: f"hidden size != heads * {HEAD_DIM}",
    -6: "packed blocks must be positive and their sum must divide the packed dimension",
    -7: "unsupported shape",
}

_lib = None


def _open(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    for name, args in _SIGS.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = _I
    return lib


def lib() -> ctypes.CDLL:
    """The loaded oracle library, built from oracle.cpp first if needed."""
    global _lib
    if _lib is None:
        _lib = _open(_build.build())
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Run the oracle from another build of its source (tests that plant a
    mistake compile a modified copy and check that a pin catches it)."""
    global _lib
    saved = lib()
    _lib = _open(path)
    try:
        yield
    finally:
        _lib = saved


def num_threads() -> int:
    """OpenMP threads the oracle computes with (its host-core count)."""
    return int(lib().oracle_num_threads())


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise ValueError(f"{name}: {_ERRORS.get(st, st)}")


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data


def _i64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


# ---------------------------------------------------------------------------
# Constraint checks ("Constraints and validation" section).
# ---------------------------------------------------------------------------

def check_degree(tp_degree: int, rank: int | None = None) -> None:
    if tp_degree < 1:
        raise ValueError(f"tp_degree must be >= 1, got {tp_degree}")
    if rank is not None and not (0 <= rank < tp_degree):
        raise ValueError(f"rank {rank} outside [0, {tp_degree})")


def check_heads(D: int, heads: int, tp_degree: int) -> None:
    _call("oracle_check_heads", D, heads, tp_degree)


# ---------------------------------------------------------------------------
# Shard slicing: index arithmetic on any dtype (bf16 bit patterns included).
# ---------------------------------------------------------------------------

def _as2d(W):
    W = np.ascontiguousarray(W)
    return (W.reshape(-1, 1) if W.ndim == 1 else W), W.ndim == 1


def slice_colwise(W, tp_degree: int, rank: int) -> np.ndarray:
    """Rows [rank*N/T, (rank+1)*N/T) of W[N, K] (also a 1-D bias)."""
    check_degree(tp_degree, rank)
    W2, flat = _as2d(W)
    rows, cols = W2.shape
    out = np.empty((rows // tp_degree if rows % tp_degree == 0 else 0, cols), dtype=W2.dtype)
    _call("oracle_slice_colwise", _p(W2), rows, cols, W2.itemsize, tp_degree, rank, _p(out))
    return out.reshape(-1) if flat else out


def slice_rowwise(W, tp_degree: int, rank: int) -> np.ndarray:
    """Columns [rank*K/T, (rank+1)*K/T) of every row of W[N, K]."""
    check_degree(tp_degree, rank)
    W = np.ascontiguousarray(W)
    rows, cols = W.shape
    out = np.empty((rows, cols // tp_degree if cols % tp_degree == 0 else 0), dtype=W.dtype)
    _call("oracle_slice_rowwise", _p(W), rows, cols, W.itemsize, tp_degree, rank, _p(out))
    return out


def packed_block_sizes(dim: int, blocks, tp_degree: int) -> list[int]:
    """Absolute block sizes of a packed dimension ("Fused projections")."""
    b = _i64(blocks)
    sizes = np.zeros(max(len(b), 1), dtype=np.int64)
    _call("oracle_packed_block_sizes", dim, _p(b) if len(b) else None, len(b), tp_degree, _p(sizes))
    return [int(s) for s in sizes[:len(b)]]


def slice_packed_colwise(W, blocks, tp_degree: int, rank: int) -> np.ndarray:
    check_degree(tp_degree, rank)
    W2, flat = _as2d(W)
    rows, cols = W2.shape
    packed_block_sizes(rows, blocks, tp_degree)
    b = _i64(blocks)
    out = np.empty((rows // tp_degree, cols), dtype=W2.dtype)
    _call("oracle_slice_packed_colwise", _p(W2), rows, cols, W2.itemsize, _p(b), len(b), tp_degree, rank, _p(out))
    return out.reshape(-1) if flat else out


def slice_packed_rowwise(W, blocks, tp_degree: int, rank: int) -> np.ndarray:
    check_degree(tp_degree, rank)
    W = np.ascontiguousarray(W)
    rows, cols = W.shape
    packed_block_sizes(cols, blocks, tp_degree)
    b = _i64(blocks)
    out = np.empty((rows, cols // tp_degree), dtype=W.dtype)
    _call("oracle_slice_packed_rowwise", _p(W), rows, cols, W.itemsize, _p(b), len(b), tp_degree, rank, _p(out))
    return out


def slice_qkv_heads(W_qkv, heads: int, tp_degree: int, rank: int) -> np.ndarray:
    """Head split of [Q; K; V] (packed colwise, blocks [1, 1, 1]): [Q_r; K_r; V_r]."""
    check_degree(tp_degree, rank)
    W = np.ascontiguousarray(W_qkv)
    rows, D = W.shape
    check_heads(D, heads, tp_degree)
    if rows != 3 * D:
        raise ValueError("W_qkv must have 3*D rows")
    out = np.empty((3 * D // tp_degree, D), dtype=W.dtype)
    _call("oracle_slice_qkv_heads", _p(W), rows, D, W.itemsize, heads, tp_degree, rank, _p(out))
    return out


# ---------------------------------------------------------------------------
# Dense pieces.
# ---------------------------------------------------------------------------

def linear(X, W, b=None) -> np.ndarray:
    """nn.Linear: Y = X W^T (+ b), W is [out_features, in_features]."""
    X, W, b = _f64(X), _f64(W), _f64(b)
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("linear: X and W disagree on in_features")
    Y = np.empty((M, N))
    _call("oracle_linear", _p(X), M, K, _p(W), N, _p(b), _p(Y))
    return Y


def gelu_tanh(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _call("oracle_gelu_tanh", _p(x), x.size, _p(y))
    return y


def silu(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _call("oracle_silu", _p(x), x.size, _p(y))
    return y


def softmax_rows(S) -> np.ndarray:
    S = _f64(S)
    P = np.empty_like(S)
    _call("oracle_softmax_rows", _p(S), S.shape[0] if S.ndim > 1 else 1, S.shape[-1], _p(P))
    return P


def sdpa(Q, K, V, scale: float | None = None, return_lse: bool = False):
    """softmax(Q K^T * scale) V for one head (scale 1/sqrt(d) by default); with
    return_lse also each row's log-sum-exp of the scaled scores."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Mq, d = Q.shape
    Mk = K.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.empty((Mq, d))
    lse = np.empty(Mq)
    _call("oracle_sdpa", _p(Q), Mq, _p(K), _p(V), Mk, d, float(scale), _p(O), _p(lse))
    return (O, lse) if return_lse else O


def attn_merge(O_parts, lse_parts):
    """Ring attention's combination of per-key-block results ("Context
    parallelism" page): O_parts [nparts, M, d] (each block's normalised
    attention output), lse_parts [nparts, M] (natural log-sum-exp of each
    block's scaled scores) -> (O [M, d], lse [M]) over all the blocks' keys."""
    Op = np.ascontiguousarray(O_parts, dtype=np.float64)
    Lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, M, d = Op.shape
    O, lse = np.empty((M, d)), np.empty(M)
    _call("oracle_attn_merge", _p(Op), _p(Lp), n, M, d, _p(O), _p(lse))
    return O, lse


def reduce_partials(parts, bias=None) -> np.ndarray:
    """sum_r Part_r (r ascending) + bias once: the AllReduce's per-element sum."""
    P = np.ascontiguousarray(np.stack([np.asarray(p, dtype=np.float64) for p in parts]))
    T, M, N = P.shape
    Y = np.empty((M, N))
    _call("oracle_reduce_partials", _p(P), T, M, N, _p(_f64(bias)), _p(Y))
    return Y


# ---------------------------------------------------------------------------
# MLP pair.  act: gelu_tanh (the layer's), or the identity (exactness pins).
# ---------------------------------------------------------------------------

def _act_code(act) -> int:
    if act is None:
        return 0
    if act is gelu_tanh:
        return 1
    probe = np.array([-1.5, 0.25, 2.0])
    if np.array_equal(np.asarray(act(probe.copy()), dtype=np.float64), probe):
        return 0
    raise ValueError("the oracle's MLP supports the tanh GELU and the identity")


def mlp_unsharded(X, W_up, b_up, W_down, b_down, act=gelu_tanh):
    X, W_up, b_up, W_down, b_down = map(_f64, (X, W_up, b_up, W_down, b_down))
    M, D = X.shape
    F = W_up.shape[0]
    Y = np.empty((M, D))
    _call("oracle_mlp_unsharded", _p(X), M, D, _p(W_up), _p(b_up), F, _p(W_down), _p(b_down), _act_code(act), _p(Y))
    return Y


def mlp_colwise_shard(X, W_up, b_up, tp_degree, rank, act=gelu_tanh):
    """H_r = act(X W_up,r^T + b_up,r) (b_up may be None)."""
    X, W_up, b_up = map(_f64, (X, W_up, b_up))
    M, D = X.shape
    F = W_up.shape[0]
    H = np.empty((M, F // tp_degree if tp_degree > 0 else 0))
    _call("oracle_mlp_colwise_shard", _p(X), M, D, _p(W_up), _p(b_up), F, tp_degree, rank, _act_code(act), _p(H))
    return H


def mlp_rowwise_partial(H_r, W_down, tp_degree, rank):
    """Part_r = H_r W_down,r^T (no bias)."""
    H, W_down = _f64(H_r), _f64(W_down)
    D, F = W_down.shape
    P = np.empty((H.shape[0], D))
    _call("oracle_mlp_rowwise_partial", _p(H), H.shape[0], _p(W_down), D, F, tp_degree, rank, _p(P))
    return P


def mlp_sharded_summed(X, W_up, b_up, W_down, b_down, tp_degree, act=gelu_tanh):
    X, W_up, b_up, W_down, b_down = map(_f64, (X, W_up, b_up, W_down, b_down))
    M, D = X.shape
    F = W_up.shape[0]
    Y = np.empty((M, D))
    _call("oracle_mlp_sharded_summed", _p(X), M, D, _p(W_up), _p(b_up), F, _p(W_down), _p(b_down), tp_degree,
          _act_code(act), _p(Y))
    return Y


def swiglu_unsharded(X, W_in, b_in, W_out, b_out):
    """W_in = [W_gate; W_up] (2F x D), b_in = [b_gate; b_up] or None."""
    X, W_in, b_in, W_out, b_out = map(_f64, (X, W_in, b_in, W_out, b_out))
    M, D = X.shape
    F = W_in.shape[0] // 2
    Y = np.empty((M, D))
    _call("oracle_swiglu_unsharded", _p(X), M, D, _p(W_in), _p(b_in), F, _p(W_out), _p(b_out), _p(Y))
    return Y


def swiglu_sharded_summed(X, W_in, b_in, W_out, b_out, tp_degree):
    X, W_in, b_in, W_out, b_out = map(_f64, (X, W_in, b_in, W_out, b_out))
    M, D = X.shape
    F = W_in.shape[0] // 2
    Y = np.empty((M, D))
    _call("oracle_swiglu_sharded_summed", _p(X), M, D, _p(W_in), _p(b_in), F, _p(W_out), _p(b_out), tp_degree, _p(Y))
    return Y


def rowwise_split_input(X, W, b, tp_degree):
    """sum_r X[:, r-th K/T block] . W_r^T (+ b once)."""
    X, W, b = map(_f64, (X, W, b))
    M, K = X.shape
    N = W.shape[0]
    Y = np.empty((M, N))
    _call("oracle_rowwise_split_input", _p(X), M, K, _p(W), N, _p(b), tp_degree, _p(Y))
    return Y


# ---------------------------------------------------------------------------
# Attention block and dual-stream joint attention.
# ---------------------------------------------------------------------------

def attn_unsharded(X, W_qkv, W_o, heads):
    X, W_qkv, W_o = map(_f64, (X, W_qkv, W_o))
    M, D = X.shape
    Y = np.empty((M, D))
    _call("oracle_attn_unsharded", _p(X), M, D, _p(W_qkv), _p(W_o), heads, _p(Y))
    return Y


def attn_shard_output(X, W_qkv, heads, tp_degree, rank):
    """O_r: shard r's attention output over its H/T heads, [M, D/T]."""
    X, W_qkv = _f64(X), _f64(W_qkv)
    M, D = X.shape
    O = np.empty((M, D // tp_degree if tp_degree > 0 else 0))
    _call("oracle_attn_shard_output", _p(X), M, D, _p(W_qkv), heads, tp_degree, rank, _p(O))
    return O


def attn_sharded_summed(X, W_qkv, W_o, heads, tp_degree):
    X, W_qkv, W_o = map(_f64, (X, W_qkv, W_o))
    M, D = X.shape
    Y = np.empty((M, D))
    _call("oracle_attn_rows", _p(X), M, D, _p(W_qkv), _p(W_o), heads, None, 0, tp_degree, _p(Y))
    return Y


def attn_rows(X, W_qkv, W_o, heads, rows, tp_degree=1):
    """Attention output at the given query rows only.  K and V need every token;
    queries are independent, so the selected rows equal those of the full output."""
    X, W_qkv, W_o = map(_f64, (X, W_qkv, W_o))
    M, D = X.shape
    r = _i64(rows)
    Y = np.empty((len(r), D))
    _call("oracle_attn_rows", _p(X), M, D, _p(W_qkv), _p(W_o), heads, _p(r), len(r), tp_degree, _p(Y))
    return Y


def joint_attn_unsharded(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads):
    """Returns (Y_img, Y_txt)."""
    Xi, Xt, Wqi, Wqt, Woi, Wot = map(_f64, (X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt))
    D = Wqi.shape[1]
    Xi, Xt = Xi.reshape(-1, D), Xt.reshape(-1, D)
    Yi, Yt = np.empty((Xi.shape[0], D)), np.empty((Xt.shape[0], D))
    _call("oracle_joint_attn_unsharded", _p(Xi), Xi.shape[0], _p(Xt), Xt.shape[0], D, _p(Wqi), _p(Wqt), _p(Woi),
          _p(Wot), heads, _p(Yi), _p(Yt))
    return Yi, Yt


def joint_attn_rows(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, rows_img, rows_txt, tp_degree=1):
    """(Y_img[rows_img], Y_txt[rows_txt]); K and V need every token of both streams."""
    Xi, Xt, Wqi, Wqt, Woi, Wot = map(_f64, (X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt))
    D = Wqi.shape[1]
    Xi, Xt = Xi.reshape(-1, D), Xt.reshape(-1, D)
    ri, rt = _i64(rows_img), _i64(rows_txt)
    Yi, Yt = np.empty((len(ri), D)), np.empty((len(rt), D))
    _call("oracle_joint_attn_rows", _p(Xi), Xi.shape[0], _p(Xt), Xt.shape[0], D, _p(Wqi), _p(Wqt), _p(Woi), _p(Wot),
          heads, _p(ri) if len(ri) else None, len(ri), _p(rt) if len(rt) else None, len(rt), tp_degree, _p(Yi),
          _p(Yt))
    return Yi, Yt


def joint_attn_sharded_summed(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, tp_degree):
    Mi = np.asarray(X_img).reshape(-1, np.asarray(W_qkv_img).shape[1]).shape[0]
    Mt = np.asarray(X_txt).reshape(-1, np.asarray(W_qkv_img).shape[1]).shape[0]
    return joint_attn_rows(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, np.arange(Mi),
                           np.arange(Mt), tp_degree)


# ---------------------------------------------------------------------------
# Composed block: Y = mlp_pair(attn_block(X)) (no residual, no norm).
# ---------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (via float32, ties to even), as float64.

    Used only where a layer's output is handed to the next layer as a bf16 tensor
    (the attention output feeding the MLP in the composed block)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32)
    u = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def block_rows(X, W_qkv, W_o, heads, W_up, b_up, W_down, b_down, rows, tp_degree=1, round_between=True):
    """Composed block at selected token rows; returns (A, Y).

    A is the attention layer's output (exact, to compare with that layer's
    result).  The tensor handed from the attention layer to the MLP pair is a
    bf16 tensor, so the MLP's input is A rounded to bf16 (``round_between``)."""
    A = attn_rows(X, W_qkv, W_o, heads, rows, tp_degree)
    A_in = round_bf16(A) if round_between else A
    return A, mlp_sharded_summed(A_in, W_up, b_up, W_down, b_down, tp_degree)
