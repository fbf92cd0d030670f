"""Python binding of libtp (include/tp.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (or raw device addresses as ints) and forwards plain pointers and
sizes through ctypes.  Nothing here computes: every step of every layer runs
in the CUDA kernels of ``libtp.so``.  If the library is missing this module
raises on first use; there is no fallback.

The convenience wrappers at the end (``mlp_pair``, ``swiglu_mlp_pair``,
``attn_block``, ``MlpPair``, ``AttnBlock``) only allocate outputs and
workspaces with torch and call the C entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp.so")

TP_COLWISE = 0
TP_ROWWISE = 1
TP_ROWWISE_SPLIT_INPUT = 2
TP_OUT_BF16 = 0
TP_OUT_F16 = 1

STATUS = {
    0: "TP_OK", 1: "TP_ERR_NULL", 2: "TP_ERR_BAD_DEGREE", 3: "TP_ERR_BAD_RANK",
    4: "TP_ERR_INDIVISIBLE", 5: "TP_ERR_HEADS_INDIVISIBLE", 6: "TP_ERR_BAD_SHAPE",
    7: "TP_ERR_ALIGNMENT", 8: "TP_ERR_WORKSPACE", 9: "TP_ERR_CUDA",
    10: "TP_ERR_DEVICE_TIMEOUT", 11: "TP_ERR_BAD_STYLE", 12: "TP_ERR_BAD_HANDLE",
    13: "TP_ERR_SCRATCH_LIMIT", 14: "TP_ERR_BAD_BLOCKS", 15: "TP_ERR_RANGE",
}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/tp.h
SIGNATURES = {
    "tp_status_string": (ctypes.c_char_p, [_I]),
    "tp_abi_version": (_I, []),
    "tp_last_error_message": (ctypes.c_char_p, []),
    "tp_check_device_error": (_I, [_P]),
    "tp_debug_watchdog": (_I, [ctypes.c_uint32, _P]),
    "tp_gemm_tile_plan": (_I, [_I64, _I64, _I, _I]),
    "tp_shard_weight": (_I, [_P, _I64, _I64, _I, _I, _I, _P, _P]),
    "tp_shard_weight_all": (_I, [_P, _I64, _I64, _I, _I, _P, _P]),
    "tp_kernel_launches": (ctypes.c_uint64, []),
    "tp_shard_qkv_heads_all": (_I, [_P, _I64, _I, _I, _P, _P]),
    "tp_shard_bias": (_I, [_P, _I64, _I, _I, _P, _P]),
    "tp_shard_qkv_heads": (_I, [_P, _I64, _I, _I, _I, _P, _P]),
    "tp_colwise_linear": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _I, _I, _P, _P]),
    "tp_rowwise_linear_sum": (_I, [_P, _I64, _I64, _P, _I64, _P, _I, _P, _P]),
    "tp_sdpa_shards": (_I, [_P, _I64, _I, _I, _P, _P]),
    "tp_reduce_partials": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "tp_mlp_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "tp_mlp_pair": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "tp_attn_workspace_bytes": (_SZ, [_I64, _I64, _I, _I]),
    "tp_attn_block": (_I, [_P, _I64, _I64, _P, _P, _I, _I, _P, _P, _SZ, _P]),
    "tp_mlp_prepare": (_I, [_P, _P, _P, _P, _I64, _I64, _I, _P, ctypes.POINTER(_P)]),
    "tp_mlp_run_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "tp_mlp_run": (_I, [_P, _P, _I64, _P, _P, _SZ, _P]),
    "tp_attn_prepare": (_I, [_P, _P, _I64, _I, _I, _P, ctypes.POINTER(_P)]),
    "tp_attn_run_workspace_bytes": (_SZ, [_I64, _I64, _I, _I]),
    "tp_attn_run": (_I, [_P, _P, _I64, _P, _P, _SZ, _P]),
    "tp_destroy": (None, [_P]),
    "tp_mlp_pair_sharded_noalloc": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _P]),
    "tp_shard_packed": (_I, [_P, _I64, _I64, _I, ctypes.POINTER(_I64), _I, _I, _I, _P, _P]),
    "tp_shard_packed_all": (_I, [_P, _I64, _I64, _I, ctypes.POINTER(_I64), _I, _I, _P, _P]),
    "tp_colwise_swiglu": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _P, _P]),
    "tp_rowwise_split_input_linear": (_I, [_P, _I64, _I64, _P, _I64, _P, _I, _P, _P]),
    "tp_swiglu_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "tp_swiglu_mlp_pair": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "tp_swiglu_prepare": (_I, [_P, _P, _P, _P, _I64, _I64, _I, _P, ctypes.POINTER(_P)]),
    "tp_joint_attn_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "tp_joint_attn_block": (_I, [_P, _I64, _P, _I64, _I64, _P, _P, _P, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "tp_joint_attn_prepare": (_I, [_P, _P, _P, _P, _I64, _I, _I, _P, ctypes.POINTER(_P)]),
    "tp_joint_attn_run_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "tp_joint_attn_run": (_I, [_P, _P, _I64, _P, _I64, _P, _P, _P, _SZ, _P]),
    "tp_colwise_linear_rows": (_I, [_P, _I64, _I64, _P, _P, _I64, _I, _I, _I, _P, _I64, _P]),
    "tp_shard_weights_batch": (_I, [_P, _I, _I, _P]),
    "tp_rowwise_linear_sum_rows": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P, _I, _P, _P]),
    "tp_sdpa_block_stats": (_I, [_P, _I64, _P, _I64, _I, _I, _P, _P, _P]),
    "tp_attn_merge": (_I, [_P, _P, _I, _I64, _I, _I, _P, _P, _P]),
    "tp_unshard_rowwise_all": (_I, [_P, _I64, _I64, _I, _P, _P]),
    "tp_mlp_rank_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "tp_mlp_rank_partial": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "tp_attn_rank_workspace_bytes": (_SZ, [_I64, _I64, _I, _I]),
    "tp_attn_rank_partial": (_I, [_P, _I64, _I64, _P, _P, _I, _I, _P, _P, _SZ, _P]),
}

_lib = None


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().tp_status_string(status).decode()
        extra = lib().tp_last_error_message().decode() if status == 9 else ""
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg}){' - ' + extra if extra else ''}")


def lib() -> ctypes.CDLL:
    """The loaded libtp.so (loaded once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m tensor_transformer_layers_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise TPError(status, where)


# --------------------------------------------------------------------------- raw entry points
def tp_status_string(status: int) -> str:
    return lib().tp_status_string(status).decode()


def tp_abi_version() -> int:
    return lib().tp_abi_version()


def tp_last_error_message() -> str:
    return lib().tp_last_error_message().decode()


def tp_check_device_error(stream=None) -> int:
    return lib().tp_check_device_error(_stream(stream))


def tp_debug_watchdog(wait_ms, stream=None) -> int:
    return lib().tp_debug_watchdog(wait_ms, _stream(stream))


GEMM_PLANS = {0: "pair256x256", 1: "cta128x256", 2: "cta128x128"}


def tp_gemm_tile_plan(M, N, groups, swiglu=False) -> int:
    return lib().tp_gemm_tile_plan(M, N, groups, int(bool(swiglu)))


def tp_shard_weight(W, rows, cols, style, tp_degree, rank, out, stream=None) -> int:
    return lib().tp_shard_weight(_ptr(W), rows, cols, style, tp_degree, rank, _ptr(out), _stream(stream))


def tp_shard_weight_all(W, rows, cols, style, tp_degree, out, stream=None) -> int:
    return lib().tp_shard_weight_all(_ptr(W), rows, cols, style, tp_degree, _ptr(out), _stream(stream))


def tp_shard_qkv_heads_all(W_qkv, D, heads, tp_degree, out, stream=None) -> int:
    return lib().tp_shard_qkv_heads_all(_ptr(W_qkv), D, heads, tp_degree, _ptr(out), _stream(stream))


def tp_kernel_launches() -> int:
    return lib().tp_kernel_launches()


def tp_shard_bias(b, n, tp_degree, rank, out, stream=None) -> int:
    return lib().tp_shard_bias(_ptr(b), n, tp_degree, rank, _ptr(out), _stream(stream))


def tp_shard_qkv_heads(W_qkv, D, heads, tp_degree, rank, out, stream=None) -> int:
    return lib().tp_shard_qkv_heads(_ptr(W_qkv), D, heads, tp_degree, rank, _ptr(out), _stream(stream))


def tp_colwise_linear(X, M, K, W_shards, b_shards, N_s, tp_degree, gelu, out_dtype, out, stream=None) -> int:
    return lib().tp_colwise_linear(_ptr(X), M, K, _ptr(W_shards), _ptr(b_shards), N_s, tp_degree,
                                   int(bool(gelu)), int(out_dtype), _ptr(out), _stream(stream))


def tp_rowwise_linear_sum(A_shards, M, K_s, W_shards, N, bias, tp_degree, Y, stream=None) -> int:
    return lib().tp_rowwise_linear_sum(_ptr(A_shards), M, K_s, _ptr(W_shards), N, _ptr(bias), tp_degree,
                                       _ptr(Y), _stream(stream))


def tp_sdpa_shards(QKV, M, heads, tp_degree, O, stream=None) -> int:
    return lib().tp_sdpa_shards(_ptr(QKV), M, heads, tp_degree, _ptr(O), _stream(stream))


def tp_reduce_partials(parts, M, N, tp_degree, bias, Y, stream=None) -> int:
    return lib().tp_reduce_partials(_ptr(parts), M, N, tp_degree, _ptr(bias), _ptr(Y), _stream(stream))


def tp_mlp_workspace_bytes(M, D, F, tp_degree) -> int:
    return lib().tp_mlp_workspace_bytes(M, D, F, tp_degree)


def tp_mlp_run_workspace_bytes(M, D, F, tp_degree) -> int:
    return lib().tp_mlp_run_workspace_bytes(M, D, F, tp_degree)


def tp_attn_workspace_bytes(M, D, heads, tp_degree) -> int:
    return lib().tp_attn_workspace_bytes(M, D, heads, tp_degree)


def tp_attn_run_workspace_bytes(M, D, heads, tp_degree) -> int:
    return lib().tp_attn_run_workspace_bytes(M, D, heads, tp_degree)


def tp_mlp_pair(X, M, D, F, W_up, b_up, W_down, b_down, tp_degree, Y, ws, ws_bytes, stream=None) -> int:
    return lib().tp_mlp_pair(_ptr(X), M, D, F, _ptr(W_up), _ptr(b_up), _ptr(W_down), _ptr(b_down), tp_degree,
                             _ptr(Y), _ptr(ws), ws_bytes, _stream(stream))


def tp_attn_block(X, M, D, W_qkv, W_o, heads, tp_degree, Y, ws, ws_bytes, stream=None) -> int:
    return lib().tp_attn_block(_ptr(X), M, D, _ptr(W_qkv), _ptr(W_o), heads, tp_degree, _ptr(Y), _ptr(ws),
                               ws_bytes, _stream(stream))


def tp_mlp_prepare(W_up, b_up, W_down, b_down, D, F, tp_degree, stream=None):
    h = _P()
    st = lib().tp_mlp_prepare(_ptr(W_up), _ptr(b_up), _ptr(W_down), _ptr(b_down), D, F, tp_degree,
                              _stream(stream), ctypes.byref(h))
    return st, h.value


def tp_mlp_run(handle, X, M, Y, ws, ws_bytes, stream=None) -> int:
    return lib().tp_mlp_run(handle, _ptr(X), M, _ptr(Y), _ptr(ws), ws_bytes, _stream(stream))


def tp_attn_prepare(W_qkv, W_o, D, heads, tp_degree, stream=None):
    h = _P()
    st = lib().tp_attn_prepare(_ptr(W_qkv), _ptr(W_o), D, heads, tp_degree, _stream(stream), ctypes.byref(h))
    return st, h.value


def tp_attn_run(handle, X, M, Y, ws, ws_bytes, stream=None) -> int:
    return lib().tp_attn_run(handle, _ptr(X), M, _ptr(Y), _ptr(ws), ws_bytes, _stream(stream))


def tp_destroy(handle) -> None:
    lib().tp_destroy(handle)


def tp_mlp_pair_sharded_noalloc(X, M, D, F, W_up_shards, b_up_shards, W_down_shards, b_down, tp_degree, Y,
                                stream=None) -> int:
    """The MLP pair on pre-sharded weights with no device allocation (fixed
    64 MiB library scratch); see include/tp.h."""
    return lib().tp_mlp_pair_sharded_noalloc(_ptr(X), M, D, F, _ptr(W_up_shards), _ptr(b_up_shards),
                                             _ptr(W_down_shards), _ptr(b_down), tp_degree, _ptr(Y),
                                             _stream(stream))


class tp_shard_job(ctypes.Structure):
    """Mirrors tp_shard_job in include/tp.h."""
    _fields_ = [("W", _P), ("rows", _I64), ("cols", _I64), ("style", _I), ("out", _P),
                ("blocks", ctypes.POINTER(_I64)), ("nblocks", _I)]


def tp_shard_weights_batch(jobs, tp_degree, stream=None) -> int:
    """jobs: list of (W, rows, cols, style, out) or (W, rows, cols, style, out, blocks);
    all sliced in one launch (up to 8 plain jobs or packed blocks)."""
    keep, items = [], []
    for job in jobs:
        W, r, c, s, o = job[:5]
        blocks = job[5] if len(job) > 5 else None
        arr, n = _blocks(blocks)
        keep.append(arr)
        items.append(tp_shard_job(_ptr(W), r, c, s, _ptr(o), ctypes.cast(arr, ctypes.POINTER(_I64)) if arr else None,
                                  n))
    table = (tp_shard_job * max(len(items), 1))(*items)
    return lib().tp_shard_weights_batch(ctypes.cast(table, _P) if items else None, len(items), tp_degree,
                                        _stream(stream))


def _blocks(blocks):
    """Host int64 array for a packed call (None stays NULL)."""
    if blocks is None:
        return None, 0
    blocks = [int(b) for b in blocks]
    return (_I64 * max(len(blocks), 1))(*blocks), len(blocks)


def tp_shard_packed(W, rows, cols, style, blocks, tp_degree, rank, out, stream=None) -> int:
    arr, n = _blocks(blocks)
    return lib().tp_shard_packed(_ptr(W), rows, cols, style, arr, n, tp_degree, rank, _ptr(out), _stream(stream))


def tp_shard_packed_all(W, rows, cols, style, blocks, tp_degree, out, stream=None) -> int:
    arr, n = _blocks(blocks)
    return lib().tp_shard_packed_all(_ptr(W), rows, cols, style, arr, n, tp_degree, _ptr(out), _stream(stream))


def tp_colwise_swiglu(X, M, K, W_shards, b_shards, F_s, tp_degree, out, stream=None) -> int:
    return lib().tp_colwise_swiglu(_ptr(X), M, K, _ptr(W_shards), _ptr(b_shards), F_s, tp_degree, _ptr(out),
                                   _stream(stream))


def tp_rowwise_split_input_linear(X, M, K, W_shards, N, bias, tp_degree, Y, stream=None) -> int:
    return lib().tp_rowwise_split_input_linear(_ptr(X), M, K, _ptr(W_shards), N, _ptr(bias), tp_degree, _ptr(Y),
                                               _stream(stream))


def tp_swiglu_workspace_bytes(M, D, F, tp_degree) -> int:
    return lib().tp_swiglu_workspace_bytes(M, D, F, tp_degree)


def tp_swiglu_mlp_pair(X, M, D, F, W_in, b_in, W_out, b_out, tp_degree, Y, ws, ws_bytes, stream=None) -> int:
    return lib().tp_swiglu_mlp_pair(_ptr(X), M, D, F, _ptr(W_in), _ptr(b_in), _ptr(W_out), _ptr(b_out), tp_degree,
                                    _ptr(Y), _ptr(ws), ws_bytes, _stream(stream))


def tp_swiglu_prepare(W_in, b_in, W_out, b_out, D, F, tp_degree, stream=None):
    h = _P()
    st = lib().tp_swiglu_prepare(_ptr(W_in), _ptr(b_in), _ptr(W_out), _ptr(b_out), D, F, tp_degree,
                                 _stream(stream), ctypes.byref(h))
    return st, h.value


def tp_colwise_linear_rows(X, M, K, W_shards, b_shards, N_s, tp_degree, gelu, out_dtype, out, out_rows,
                           stream=None) -> int:
    return lib().tp_colwise_linear_rows(_ptr(X), M, K, _ptr(W_shards), _ptr(b_shards), N_s, tp_degree,
                                        int(bool(gelu)), int(out_dtype), _ptr(out), out_rows, _stream(stream))


def tp_rowwise_linear_sum_rows(A_shards, M, K_s, a_rows, W_shards, N, bias, tp_degree, Y, stream=None) -> int:
    return lib().tp_rowwise_linear_sum_rows(_ptr(A_shards), M, K_s, a_rows, _ptr(W_shards), N, _ptr(bias),
                                            tp_degree, _ptr(Y), _stream(stream))


def tp_joint_attn_workspace_bytes(M_img, M_txt, D, heads, tp_degree) -> int:
    return lib().tp_joint_attn_workspace_bytes(M_img, M_txt, D, heads, tp_degree)


def tp_joint_attn_run_workspace_bytes(M_img, M_txt, D, heads, tp_degree) -> int:
    return lib().tp_joint_attn_run_workspace_bytes(M_img, M_txt, D, heads, tp_degree)


def tp_joint_attn_block(X_img, M_img, X_txt, M_txt, D, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, tp_degree,
                        Y_img, Y_txt, ws, ws_bytes, stream=None) -> int:
    return lib().tp_joint_attn_block(_ptr(X_img), M_img, _ptr(X_txt), M_txt, D, _ptr(W_qkv_img), _ptr(W_qkv_txt),
                                     _ptr(W_o_img), _ptr(W_o_txt), heads, tp_degree, _ptr(Y_img), _ptr(Y_txt),
                                     _ptr(ws), ws_bytes, _stream(stream))


def tp_joint_attn_prepare(W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, D, heads, tp_degree, stream=None):
    h = _P()
    st = lib().tp_joint_attn_prepare(_ptr(W_qkv_img), _ptr(W_qkv_txt), _ptr(W_o_img), _ptr(W_o_txt), D, heads,
                                     tp_degree, _stream(stream), ctypes.byref(h))
    return st, h.value


def tp_joint_attn_run(handle, X_img, M_img, X_txt, M_txt, Y_img, Y_txt, ws, ws_bytes, stream=None) -> int:
    return lib().tp_joint_attn_run(handle, _ptr(X_img), M_img, _ptr(X_txt), M_txt, _ptr(Y_img), _ptr(Y_txt),
                                   _ptr(ws), ws_bytes, _stream(stream))


# --------------------------------------------------------------------------- convenience
def tp_sdpa_block_stats(Q_qkv, Mq, KV_qkv, Mk, heads, tp_degree, O, lse, stream=None) -> int:
    return lib().tp_sdpa_block_stats(_ptr(Q_qkv), Mq, _ptr(KV_qkv), Mk, heads, tp_degree, _ptr(O), _ptr(lse),
                                     _stream(stream))


def tp_attn_merge(O_parts, lse_parts, nparts, M, heads, tp_degree, O, lse_out=None, stream=None) -> int:
    return lib().tp_attn_merge(_ptr(O_parts), _ptr(lse_parts), nparts, M, heads, tp_degree, _ptr(O), _ptr(lse_out),
                               _stream(stream))


def tp_unshard_rowwise_all(src, rows, cols, tp_degree, out, stream=None) -> int:
    return lib().tp_unshard_rowwise_all(_ptr(src), rows, cols, tp_degree, _ptr(out), _stream(stream))


def tp_mlp_rank_workspace_bytes(M, D, F, tp_degree) -> int:
    return lib().tp_mlp_rank_workspace_bytes(M, D, F, tp_degree)


def tp_mlp_rank_partial(X, M, D, F, W_up_r, b_up_r, W_down_r, tp_degree, part, ws, ws_bytes, stream=None) -> int:
    return lib().tp_mlp_rank_partial(_ptr(X), M, D, F, _ptr(W_up_r), _ptr(b_up_r), _ptr(W_down_r), tp_degree,
                                     _ptr(part), _ptr(ws), ws_bytes, _stream(stream))


def tp_attn_rank_workspace_bytes(M, D, heads, tp_degree) -> int:
    return lib().tp_attn_rank_workspace_bytes(M, D, heads, tp_degree)


def tp_attn_rank_partial(X, M, D, W_qkv_r, W_o_r, heads, tp_degree, part, ws, ws_bytes, stream=None) -> int:
    return lib().tp_attn_rank_partial(_ptr(X), M, D, _ptr(W_qkv_r), _ptr(W_o_r), heads, tp_degree, _ptr(part),
                                      _ptr(ws), ws_bytes, _stream(stream))


def _u16(t: torch.Tensor) -> torch.Tensor:
    """bf16 bit patterns travel as 16-bit tensors; accept bfloat16 or int16/uint16 storage."""
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16, torch.float16):
        raise TypeError(f"expected a 16-bit tensor of bf16 values, got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def mlp_pair(X, W_up, b_up, W_down, b_down, tp_degree: int, stream=None) -> torch.Tensor:
    """One-shot MLP pair (slices the weights, then runs); returns Y [M, D] (bf16)."""
    _u16(X), _u16(W_up), _u16(W_down)
    M, D = X.shape
    F = W_up.shape[0]
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=X.device)
    nb = tp_mlp_workspace_bytes(M, D, F, tp_degree)
    ws = _workspace(nb, X.device)
    _check(tp_mlp_pair(X, M, D, F, W_up, b_up, W_down, b_down, tp_degree, Y, ws, nb, stream), "tp_mlp_pair")
    return Y


def swiglu_mlp_pair(X, W_in, b_in, W_out, b_out, tp_degree: int, stream=None) -> torch.Tensor:
    """One-shot SwiGLU pair, W_in = [W_gate; W_up]; returns Y [M, D] (bf16)."""
    _u16(X), _u16(W_in), _u16(W_out)
    M, D = X.shape
    F = W_in.shape[0] // 2
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=X.device)
    nb = tp_swiglu_workspace_bytes(M, D, F, tp_degree)
    ws = _workspace(nb, X.device)
    _check(tp_swiglu_mlp_pair(X, M, D, F, W_in, b_in, W_out, b_out, tp_degree, Y, ws, nb, stream),
           "tp_swiglu_mlp_pair")
    return Y


def attn_block(X, W_qkv, W_o, heads: int, tp_degree: int, stream=None) -> torch.Tensor:
    """One-shot attention block; returns Y [M, D] (bf16)."""
    _u16(X), _u16(W_qkv), _u16(W_o)
    M, D = X.shape
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=X.device)
    nb = tp_attn_workspace_bytes(M, D, heads, tp_degree)
    ws = _workspace(nb, X.device)
    _check(tp_attn_block(X, M, D, W_qkv, W_o, heads, tp_degree, Y, ws, nb, stream), "tp_attn_block")
    return Y


def joint_attn_block(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads: int, tp_degree: int,
                     stream=None):
    """One-shot dual-stream joint attention; returns (Y_img, Y_txt) (bf16)."""
    for t in (X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt):
        _u16(t)
    Mi, D = X_img.shape
    Mt = X_txt.shape[0]
    Yi = torch.empty((Mi, D), dtype=torch.bfloat16, device=X_img.device)
    Yt = torch.empty((Mt, D), dtype=torch.bfloat16, device=X_img.device)
    nb = tp_joint_attn_workspace_bytes(Mi, Mt, D, heads, tp_degree)
    ws = _workspace(nb, X_img.device)
    _check(tp_joint_attn_block(X_img, Mi, X_txt, Mt, D, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, tp_degree,
                               Yi, Yt, ws, nb, stream), "tp_joint_attn_block")
    return Yi, Yt


class MlpPair:
    """Shards once (tp_mlp_prepare, or tp_swiglu_prepare with
    activation="swiglu" and W_up = [W_gate; W_up]), runs many times (tp_mlp_run)."""

    def __init__(self, W_up, b_up, W_down, b_down, tp_degree: int, stream=None, activation: str = "gelu"):
        self.D = W_up.shape[1]
        self.T = tp_degree
        self.handle = None
        if activation == "gelu":
            self.F = W_up.shape[0]
            st, self.handle = tp_mlp_prepare(W_up, b_up, W_down, b_down, self.D, self.F, tp_degree, stream)
            _check(st, "tp_mlp_prepare")
        elif activation == "swiglu":
            self.F = W_up.shape[0] // 2
            st, self.handle = tp_swiglu_prepare(W_up, b_up, W_down, b_down, self.D, self.F, tp_degree, stream)
            _check(st, "tp_swiglu_prepare")
        else:
            raise ValueError(f"unknown activation {activation!r}")
        self._ws = None

    def workspace(self, M, device):
        nb = tp_mlp_run_workspace_bytes(M, self.D, self.F, self.T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = _workspace(nb, device)
        return self._ws, nb

    def __call__(self, X, Y=None, stream=None) -> torch.Tensor:
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.D), dtype=torch.bfloat16, device=X.device)
        ws, nb = self.workspace(M, X.device)
        _check(tp_mlp_run(self.handle, X, M, Y, ws, nb, stream), "tp_mlp_run")
        return Y

    def close(self):
        if self.handle:
            tp_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass


class AttnBlock:
    """Shards once (tp_attn_prepare), runs many times (tp_attn_run)."""

    def __init__(self, W_qkv, W_o, heads: int, tp_degree: int, stream=None):
        self.D = W_qkv.shape[1]
        self.heads = heads
        self.T = tp_degree
        st, self.handle = tp_attn_prepare(W_qkv, W_o, self.D, heads, tp_degree, stream)
        _check(st, "tp_attn_prepare")
        self._ws = None

    def workspace(self, M, device):
        nb = tp_attn_run_workspace_bytes(M, self.D, self.heads, self.T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = _workspace(nb, device)
        return self._ws, nb

    def __call__(self, X, Y=None, stream=None) -> torch.Tensor:
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.D), dtype=torch.bfloat16, device=X.device)
        ws, nb = self.workspace(M, X.device)
        _check(tp_attn_run(self.handle, X, M, Y, ws, nb, stream), "tp_attn_run")
        return Y

    def close(self):
        if self.handle:
            tp_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001
            pass


class JointAttnBlock:
    """Shards once (tp_joint_attn_prepare), runs many times (tp_joint_attn_run)."""

    def __init__(self, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads: int, tp_degree: int, stream=None):
        self.D = W_qkv_img.shape[1]
        self.heads = heads
        self.T = tp_degree
        self.handle = None
        st, self.handle = tp_joint_attn_prepare(W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, self.D, heads, tp_degree,
                                                stream)
        _check(st, "tp_joint_attn_prepare")
        self._ws = None

    def __call__(self, X_img, X_txt, stream=None):
        Mi, Mt = X_img.shape[0], X_txt.shape[0]
        Yi = torch.empty((Mi, self.D), dtype=torch.bfloat16, device=X_img.device)
        Yt = torch.empty((Mt, self.D), dtype=torch.bfloat16, device=X_img.device)
        nb = tp_joint_attn_run_workspace_bytes(Mi, Mt, self.D, self.heads, self.T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = _workspace(nb, X_img.device)
        _check(tp_joint_attn_run(self.handle, X_img, Mi, X_txt, Mt, Yi, Yt, self._ws, nb, stream),
               "tp_joint_attn_run")
        return Yi, Yt

    def close(self):
        if self.handle:
            tp_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001
            pass
