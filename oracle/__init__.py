"""fp64 CPU oracle for the tensor-parallel (TP) layer pair.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (``tensor_transformer_layers_b200``); the two meet only in
the seeded input generator ``synthetic``.

What it computes, and where that is defined (Diffusers documentation,
"Tensor parallelism" page, Portuguese "main" edition and Chinese v0.43.0
edition, which state the same facts):

* Opening paragraph: each device holds a column-wise or row-wise slice of a
  layer's weight and computes a partial result; the partials are combined at
  the layer boundary (by the AllReduce of a colwise->rowwise pair).
* Section "Colwise and rowwise", style table: ``colwise`` shards the output
  features (weight dim 0) and each rank computes a slice of the output;
  ``rowwise`` shards the input features (weight dim 1) and each rank computes
  a partial sum.  The paragraph under the table: a colwise projection leaves
  its output sharded, the rowwise projection that follows consumes the shard
  directly, and a single AllReduce at the block boundary rebuilds the result.
  The next paragraph: colwise Q, K, V give each rank a subset of the heads, so
  the degree must divide the head count.
* Section "Fused projections": when one Linear packs several logical tensors
  along the sharded dimension, each packed block is sharded on its own
  (a fused Q/K/V projection is packed with blocks [1, 1, 1]).
* Section "Constraints and validation": the degree must divide the head
  count, every packed block must be divisible by the degree on its own, both
  checked before any weight is split; and a plan is validated by comparing the
  single-device output with the sharded output.

Because sharding changes only where the arithmetic happens, the sharded layer
reaches exactly (up to rounding order) the unsharded layer.  The oracle is
therefore the plain definition of each layer written out in float64, with
numpy's matmul as the only library primitive.  Readings where the pages are
silent (all stated again where used):

* GELU is the tanh form 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
  (Hendrycks & Gimpel, 2016), evaluated with numpy's float64 tanh.
* A rowwise bias is added once, after the sum over shards; a colwise bias is
  sliced like weight dim 0.
* A fused QKV weight is [Q; K; V] stacked on dim 0, D rows each, head h at
  rows h*d .. h*d+d-1 inside each block; a shard's packed slice is
  [Q_r; K_r; V_r].
* Attention is softmax(Q K^T / sqrt(d)) V per head, non-causal, no mask, no
  bias, computed with a two-pass softmax (row max subtracted before exp).
* The composed block is mlp_pair(attn_block(X)), with no residual or norm.
* Sums over shards run in ascending shard order.
"""
from __future__ import annotations

import numpy as np

HEAD_DIM = 128


# ---------------------------------------------------------------------------
# Constraint checks ("Constraints and validation" section).  Raised before any
# slicing, like the pages' loader does.
# ---------------------------------------------------------------------------

def check_degree(tp_degree: int, rank: int | None = None) -> None:
    if tp_degree < 1:
        raise ValueError(f"tp_degree must be >= 1, got {tp_degree}")
    if rank is not None and not (0 <= rank < tp_degree):
        raise ValueError(f"rank {rank} outside [0, {tp_degree})")


def check_divisible(n: int, tp_degree: int, what: str) -> None:
    if n % tp_degree != 0:
        raise ValueError(f"{what}={n} is not divisible by tp_degree={tp_degree}")


def check_heads(D: int, heads: int, tp_degree: int) -> None:
    if heads % tp_degree != 0:
        raise ValueError(f"tp_degree={tp_degree} does not divide heads={heads}")
    if D != heads * HEAD_DIM:
        raise ValueError(f"hidden size {D} != heads*{HEAD_DIM}")


# ---------------------------------------------------------------------------
# Shard slicing (style table: colwise = weight dim 0, rowwise = weight dim 1).
# Pure index arithmetic; works on any dtype, bf16 bit patterns included.
# ---------------------------------------------------------------------------

def slice_colwise(W: np.ndarray, tp_degree: int, rank: int) -> np.ndarray:
    """Rows [rank*N/T, (rank+1)*N/T) of W[N, K] (also used for a 1-D bias)."""
    check_degree(tp_degree, rank)
    n = W.shape[0]
    check_divisible(n, tp_degree, "output features")
    step = n // tp_degree
    return W[rank * step:(rank + 1) * step].copy()


def slice_rowwise(W: np.ndarray, tp_degree: int, rank: int) -> np.ndarray:
    """Columns [rank*K/T, (rank+1)*K/T) of every row of W[N, K]."""
    check_degree(tp_degree, rank)
    k = W.shape[1]
    check_divisible(k, tp_degree, "input features")
    step = k // tp_degree
    return W[:, rank * step:(rank + 1) * step].copy()


def packed_block_sizes(dim: int, blocks: list[int], tp_degree: int) -> list[int]:
    """Absolute block sizes of a packed dimension ("Fused projections" section).

    ``blocks`` are proportional integers whose sum must divide the packed
    dimension ([1, 1] for equal SwiGLU gate/up halves, [1, 1, 1, 3, 3] for a
    fused Q, K, V, gate, up with mlp_ratio 3); absolute sizes, as stored on a
    Linear, are the case where the sum equals the dimension.  Every block must
    be divisible by the degree on its own, not only their sum ("Constraints and
    validation" section)."""
    if not blocks or any(b < 1 for b in blocks):
        raise ValueError("packed blocks must be positive")
    total = sum(blocks)
    if dim % total != 0:
        raise ValueError(f"sum of blocks {total} does not divide the packed dimension {dim}")
    sizes = [b * (dim // total) for b in blocks]
    for s in sizes:
        check_divisible(s, tp_degree, "packed block")
    return sizes


def slice_packed_colwise(W: np.ndarray, blocks: list[int], tp_degree: int, rank: int) -> np.ndarray:
    """Packed colwise ("Fused projections" section): W's dim 0 is split into
    consecutive blocks (proportions ``blocks``); each block is sliced colwise on
    its own and the per-block slices are stacked in block order."""
    check_degree(tp_degree, rank)
    sizes = packed_block_sizes(W.shape[0], blocks, tp_degree)
    parts, start = [], 0
    for b in sizes:
        parts.append(slice_colwise(W[start:start + b], tp_degree, rank))
        start += b
    return np.concatenate(parts, axis=0)


def slice_packed_rowwise(W: np.ndarray, blocks: list[int], tp_degree: int, rank: int) -> np.ndarray:
    """Packed rowwise: W's dim 1 is split into consecutive blocks; each block is
    sliced rowwise on its own and the per-block slices are concatenated along
    dim 1 in block order."""
    check_degree(tp_degree, rank)
    sizes = packed_block_sizes(W.shape[1], blocks, tp_degree)
    parts, start = [], 0
    for b in sizes:
        parts.append(slice_rowwise(W[:, start:start + b], tp_degree, rank))
        start += b
    return np.concatenate(parts, axis=1)


def slice_qkv_heads(W_qkv: np.ndarray, heads: int, tp_degree: int, rank: int) -> np.ndarray:
    """Head split of a fused [Q; K; V] weight: packed colwise with blocks [1, 1, 1].

    Shard ``rank`` gets heads [rank*H/T, (rank+1)*H/T) of each of Q, K and V,
    stacked as [Q_r; K_r; V_r] (3*D/T rows)."""
    D = W_qkv.shape[1]
    check_degree(tp_degree, rank)
    check_heads(D, heads, tp_degree)
    if W_qkv.shape[0] != 3 * D:
        raise ValueError("W_qkv must have 3*D rows")
    return slice_packed_colwise(W_qkv, [D, D, D], tp_degree, rank)


# ---------------------------------------------------------------------------
# Dense pieces.
# ---------------------------------------------------------------------------

def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """tanh-form GELU (Hendrycks & Gimpel 2016), float64."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def linear(X: np.ndarray, W: np.ndarray, b: np.ndarray | None = None) -> np.ndarray:
    """nn.Linear convention: Y = X W^T (+ b), W is [out_features, in_features]."""
    Y = np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    if b is not None:
        Y = Y + np.asarray(b, dtype=np.float64)[None, :]
    return Y


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Two-pass softmax over the last axis: subtract the row max, exp, divide by the sum."""
    S = np.asarray(S, dtype=np.float64)
    E = np.exp(S - S.max(axis=-1, keepdims=True))
    return E / E.sum(axis=-1, keepdims=True)


def sdpa(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float | None = None) -> np.ndarray:
    """softmax(Q K^T * scale) V for one head; Q[Mq,d], K[Mk,d], V[Mk,d]; scale 1/sqrt(d)."""
    if scale is None:
        scale = 1.0 / np.sqrt(Q.shape[1])
    return softmax_rows((Q @ K.T) * scale) @ V


def reduce_partials(parts, bias: np.ndarray | None = None) -> np.ndarray:
    """The sum an AllReduce performs at the block boundary: sum_r Part_r (r ascending), plus
    the rowwise bias once."""
    Y = np.zeros_like(np.asarray(parts[0], dtype=np.float64))
    for p in parts:
        Y = Y + np.asarray(p, dtype=np.float64)
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return Y


# ---------------------------------------------------------------------------
# MLP pair: colwise FFN-in (+bias, GELU) -> rowwise FFN-out (+bias once).
# ---------------------------------------------------------------------------

def mlp_unsharded(X, W_up, b_up, W_down, b_down, act=gelu_tanh):
    return linear(act(linear(X, W_up, b_up)), W_down, b_down)


def mlp_colwise_shard(X, W_up, b_up, tp_degree, rank, act=gelu_tanh):
    """H_r = act(X W_up,r^T + b_up,r): shard r's slice of the FFN hidden activations (b_up may be None)."""
    b_r = None if b_up is None else slice_colwise(b_up, tp_degree, rank)
    return act(linear(X, slice_colwise(W_up, tp_degree, rank), b_r))


def mlp_rowwise_partial(H_r, W_down, tp_degree, rank):
    """Part_r = H_r W_down,r^T: shard r's partial sum of the FFN output (no bias)."""
    return linear(H_r, slice_rowwise(W_down, tp_degree, rank))


def mlp_sharded_summed(X, W_up, b_up, W_down, b_down, tp_degree, act=gelu_tanh):
    check_degree(tp_degree)
    check_divisible(W_up.shape[0], tp_degree, "F")
    parts = []
    for r in range(tp_degree):
        H_r = mlp_colwise_shard(X, W_up, b_up, tp_degree, r, act)
        parts.append(mlp_rowwise_partial(H_r, W_down, tp_degree, r))
    return reduce_partials(parts, b_down)


# ---------------------------------------------------------------------------
# SwiGLU MLP pair: packed colwise [gate; up] (blocks [1, 1]) -> silu(gate) * up
# -> rowwise FFN-out.  The packed form is the pages' SwiGLU example in the
# "Fused projections" section; SiLU(x) = x * sigmoid(x) (Elfwing et al., 2018;
# SwiGLU: Shazeer, 2020).
# ---------------------------------------------------------------------------

def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu_unsharded(X, W_in, b_in, W_out, b_out):
    """W_in = [W_gate; W_up] (2F x D), b_in = [b_gate; b_up] or None."""
    F = W_in.shape[0] // 2
    G = linear(X, W_in[:F], None if b_in is None else b_in[:F])
    U = linear(X, W_in[F:], None if b_in is None else b_in[F:])
    return linear(silu(G) * U, W_out, b_out)


def swiglu_sharded_summed(X, W_in, b_in, W_out, b_out, tp_degree):
    check_degree(tp_degree)
    parts = []
    for r in range(tp_degree):
        Wr = slice_packed_colwise(W_in, [1, 1], tp_degree, r)  # [gate_r; up_r]
        Fr = Wr.shape[0] // 2
        br = None if b_in is None else slice_packed_colwise(b_in, [1, 1], tp_degree, r)
        G = linear(X, Wr[:Fr], None if br is None else br[:Fr])
        U = linear(X, Wr[Fr:], None if br is None else br[Fr:])
        parts.append(linear(silu(G) * U, slice_rowwise(W_out, tp_degree, r)))
    return reduce_partials(parts, b_out)


# ---------------------------------------------------------------------------
# rowwise_split_input (style table): a rowwise projection whose input is
# replicated; each rank takes its slice of the input's features itself.
# ---------------------------------------------------------------------------

def rowwise_split_input(X, W, b, tp_degree):
    """sum_r X[:, r-th K/T block] . W_r^T (+ b once)."""
    check_degree(tp_degree)
    parts = [linear(slice_rowwise(X, tp_degree, r), slice_rowwise(W, tp_degree, r)) for r in range(tp_degree)]
    return reduce_partials(parts, b)


# ---------------------------------------------------------------------------
# Attention block: head-split QKV (colwise) -> per-shard SDPA -> rowwise W_o.
# ---------------------------------------------------------------------------

def _heads_attention(Qs, Ks, Vs, n_heads):
    """Per-head SDPA on column blocks of width HEAD_DIM; returns concat_h O_h."""
    outs = []
    for h in range(n_heads):
        c = slice(h * HEAD_DIM, (h + 1) * HEAD_DIM)
        outs.append(sdpa(Qs[:, c], Ks[:, c], Vs[:, c]))
    return np.concatenate(outs, axis=1)


def attn_unsharded(X, W_qkv, W_o, heads):
    D = W_qkv.shape[1]
    check_heads(D, heads, 1)
    QKV = linear(X, W_qkv)
    O = _heads_attention(QKV[:, :D], QKV[:, D:2 * D], QKV[:, 2 * D:], heads)
    return linear(O, W_o)


def attn_shard_output(X, W_qkv, heads, tp_degree, rank):
    """O_r: shard r's attention output over its H/T heads, [M, D/T]."""
    D = W_qkv.shape[1]
    Dr = D // tp_degree
    QKV_r = linear(X, slice_qkv_heads(W_qkv, heads, tp_degree, rank))
    return _heads_attention(QKV_r[:, :Dr], QKV_r[:, Dr:2 * Dr], QKV_r[:, 2 * Dr:], heads // tp_degree)


def attn_sharded_summed(X, W_qkv, W_o, heads, tp_degree):
    D = W_qkv.shape[1]
    check_degree(tp_degree)
    check_heads(D, heads, tp_degree)
    parts = []
    for r in range(tp_degree):
        O_r = attn_shard_output(X, W_qkv, heads, tp_degree, r)
        parts.append(linear(O_r, slice_rowwise(W_o, tp_degree, r)))
    return reduce_partials(parts)


def attn_rows(X, W_qkv, W_o, heads, rows, tp_degree=1):
    """Attention output at the given query rows only.  K and V need every token;
    queries are independent, so the selected rows equal those of the full output."""
    D = W_qkv.shape[1]
    check_heads(D, heads, tp_degree)
    rows = np.asarray(rows)
    parts = []
    for r in range(tp_degree):
        W_r = slice_qkv_heads(W_qkv, heads, tp_degree, r)
        Dr = D // tp_degree
        Q = linear(X[rows], W_r[:Dr])
        K = linear(X, W_r[Dr:2 * Dr])
        V = linear(X, W_r[2 * Dr:])
        O_r = _heads_attention(Q, K, V, heads // tp_degree)
        parts.append(linear(O_r, slice_rowwise(W_o, tp_degree, r)))
    return reduce_partials(parts)


# ---------------------------------------------------------------------------
# Dual-stream joint attention: the image stream (to_q/k/v, to_out) and the
# text stream (add_q/k/v_proj, to_add_out) are sharded alike (the page's note
# that the encoder-stream projections follow the image-stream pattern); the
# two streams' Q, K, V are concatenated along tokens (image first, then text)
# and attended jointly; each stream's rows go through its own out-projection.
# ---------------------------------------------------------------------------

def joint_attn_unsharded(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads):
    """Returns (Y_img, Y_txt)."""
    D = W_qkv_img.shape[1]
    check_heads(D, heads, 1)
    QKV = np.concatenate([linear(X_img, W_qkv_img), linear(X_txt, W_qkv_txt)], axis=0)
    O = _heads_attention(QKV[:, :D], QKV[:, D:2 * D], QKV[:, 2 * D:], heads)
    Mi = X_img.shape[0]
    return linear(O[:Mi], W_o_img), linear(O[Mi:], W_o_txt)


def joint_attn_sharded_summed(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, tp_degree):
    D = W_qkv_img.shape[1]
    check_degree(tp_degree)
    check_heads(D, heads, tp_degree)
    Dr, Mi = D // tp_degree, X_img.shape[0]
    parts_img, parts_txt = [], []
    for r in range(tp_degree):
        QKV_r = np.concatenate([linear(X_img, slice_qkv_heads(W_qkv_img, heads, tp_degree, r)),
                                linear(X_txt, slice_qkv_heads(W_qkv_txt, heads, tp_degree, r))], axis=0)
        O_r = _heads_attention(QKV_r[:, :Dr], QKV_r[:, Dr:2 * Dr], QKV_r[:, 2 * Dr:], heads // tp_degree)
        parts_img.append(linear(O_r[:Mi], slice_rowwise(W_o_img, tp_degree, r)))
        parts_txt.append(linear(O_r[Mi:], slice_rowwise(W_o_txt, tp_degree, r)))
    return reduce_partials(parts_img), reduce_partials(parts_txt)


def joint_attn_rows(X_img, X_txt, W_qkv_img, W_qkv_txt, W_o_img, W_o_txt, heads, rows_img, rows_txt,
                    tp_degree=1):
    """(Y_img[rows_img], Y_txt[rows_txt]): K and V need every token of both
    streams; queries are independent, so these rows equal the full output's."""
    D = W_qkv_img.shape[1]
    check_heads(D, heads, tp_degree)
    Dr = D // tp_degree
    rows_img, rows_txt = np.asarray(rows_img, dtype=np.int64), np.asarray(rows_txt, dtype=np.int64)
    parts_img, parts_txt = [], []
    for r in range(tp_degree):
        Wi = slice_qkv_heads(W_qkv_img, heads, tp_degree, r)
        Wt = slice_qkv_heads(W_qkv_txt, heads, tp_degree, r)
        Q = np.concatenate([linear(X_img[rows_img], Wi[:Dr]), linear(X_txt[rows_txt], Wt[:Dr])], axis=0)
        K = np.concatenate([linear(X_img, Wi[Dr:2 * Dr]), linear(X_txt, Wt[Dr:2 * Dr])], axis=0)
        V = np.concatenate([linear(X_img, Wi[2 * Dr:]), linear(X_txt, Wt[2 * Dr:])], axis=0)
        O_r = _heads_attention(Q, K, V, heads // tp_degree)
        n = len(rows_img)
        parts_img.append(linear(O_r[:n], slice_rowwise(W_o_img, tp_degree, r)))
        parts_txt.append(linear(O_r[n:], slice_rowwise(W_o_txt, tp_degree, r)))
    return reduce_partials(parts_img), reduce_partials(parts_txt)


# ---------------------------------------------------------------------------
# Composed block: Y = mlp_pair(attn_block(X)) (no residual, no norm).
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
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
