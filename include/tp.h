/*
 * tp.h - C ABI of libtp, the B200 (sm_100a) tensor-parallel layer-pair library.
 *
 * What the library computes is defined on the Diffusers documentation page
 * "Tensor parallelism" (Portuguese "main" edition; Chinese v0.43.0 edition):
 *
 *   - opening paragraph: each device holds a column-wise ("colwise") or
 *     row-wise ("rowwise") slice of a layer's weight and computes a partial
 *     result; the partials are combined at the layer boundary;
 *   - section "Colwise and rowwise", style table: colwise shards the output
 *     features (weight dim 0), each rank computing a slice of the output;
 *     rowwise shards the input features (weight dim 1), each rank computing a
 *     partial sum; the paragraph below it: a colwise projection followed by a
 *     rowwise one needs a single AllReduce at the block boundary, and colwise
 *     Q/K/V give each rank a subset of the heads;
 *   - section "Fused projections": a Linear that packs several tensors along
 *     the sharded dimension is sharded block by block (Q/K/V: blocks [1,1,1]);
 *   - section "Fused projections" also gives the SwiGLU gate/up pair packed
 *     with blocks [1, 1], proportional blocks (e.g. [1, 1, 1, 3, 3]) or
 *     absolute sizes stored on the Linear, and packed rowwise;
 *   - style table, third row: "rowwise_split_input", a rowwise projection
 *     whose input is replicated, each rank slicing its part of the input;
 *   - the note after the style table: the encoder (text) stream's projections
 *     (add_q_proj, to_add_out, ...) follow the image stream's pattern, which
 *     with joint attention over both streams' tokens is the dual-stream block;
 *   - section "Constraints and validation": the degree must divide the head
 *     count and every packed block, checked before any weight is split.
 *
 * Here all tp_degree shards live on ONE GPU: every shard's slice is
 * materialised, each shard runs its own colwise GEMM, and the sum that the
 * AllReduce would perform is accumulated inside the rowwise GEMM (one fp32
 * accumulator walks every shard's K range), plus the rowwise bias once.
 *
 * Conventions for every entry point
 *   - Tensors are row-major.  bf16 values travel as uint16_t bit patterns.
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device,
 *     owned by the caller, and must be 16-byte aligned.  Workspaces must be
 *     256-byte aligned.  Weights are nn.Linear-shaped: [out_features x in_features].
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued on it and the call returns without waiting.
 *   - Every argument check runs before anything is launched; a call that
 *     returns an error has written nothing and launched nothing.  There is no
 *     fallback path of any kind: an unsupported shape is an error.
 *   - A returned TP_OK covers argument checks and launch errors.  A kernel's
 *     own watchdog (every wait is bounded; a wait that runs out records an
 *     error and the kernel exits) is reported by tp_check_device_error().
 */
#ifndef TP_B200_TP_H_
#define TP_B200_TP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TP_ABI_VERSION 1
#define TP_HEAD_DIM 128

typedef enum {
  TP_OK = 0,
  TP_ERR_NULL = 1,               /* a required pointer is NULL */
  TP_ERR_BAD_DEGREE = 2,         /* tp_degree < 1 */
  TP_ERR_BAD_RANK = 3,           /* rank outside [0, tp_degree) */
  TP_ERR_INDIVISIBLE = 4,        /* a sharded dimension (or packed block) % tp_degree != 0 */
  TP_ERR_HEADS_INDIVISIBLE = 5,  /* heads % tp_degree != 0 */
  TP_ERR_BAD_SHAPE = 6,          /* negative/zero size, D != heads*128, size above the supported range */
  TP_ERR_ALIGNMENT = 7,          /* pointer not 16-byte aligned, or a shard row not a multiple of 16 bytes */
  TP_ERR_WORKSPACE = 8,          /* workspace NULL, too small or not 256-byte aligned */
  TP_ERR_CUDA = 9,               /* a CUDA runtime/driver call failed (launch, tensor map, ...) */
  TP_ERR_DEVICE_TIMEOUT = 10,    /* a kernel's bounded wait ran out (see tp_check_device_error) */
  TP_ERR_BAD_STYLE = 11,         /* unknown tp_style */
  TP_ERR_BAD_HANDLE = 12,        /* NULL or foreign handle */
  TP_ERR_SCRATCH_LIMIT = 13,     /* problem too large for the no-allocation entry point's fixed scratch */
  TP_ERR_BAD_BLOCKS = 14,        /* packed blocks: count outside 1..64, a block < 1, or sum not dividing the dim */
  TP_ERR_RANGE = 15              /* an fp16 activation (e.g. the Q/K/V feeding attention) was outside the fp16
                                    range or NaN; reported by tp_check_device_error */
} tp_status;

typedef enum {
  TP_COLWISE = 0,             /* slice output features: rows [r*N/T, (r+1)*N/T) of W[N x K] */
  TP_ROWWISE = 1,             /* slice input features: columns [r*K/T, (r+1)*K/T) of every row */
  TP_ROWWISE_SPLIT_INPUT = 2  /* weight sliced as TP_ROWWISE; the replicated input is sliced by
                                 tp_rowwise_split_input_linear itself */
} tp_style;

/* Storage type of a 16-bit activation output. */
typedef enum {
  TP_OUT_BF16 = 0,
  TP_OUT_F16 = 1
} tp_out_dtype;

/* Human-readable name of a status code (static storage). */
const char* tp_status_string(int status);
int tp_abi_version(void);

/* Text describing the last CUDA failure seen by this thread inside the library
 * (the failing call and the CUDA error name), or "" if none.  Thread-local,
 * overwritten by the next failure; useful after a TP_ERR_CUDA. */
const char* tp_last_error_message(void);

/* Number of kernels this library has launched in this process (all devices,
 * all threads); a telemetry counter for benchmarks. */
uint64_t tp_kernel_launches(void);

/* Failure-detection check: launches one CTA that waits, through the same
 * bounded wait every kernel here uses, on an mbarrier that nothing arrives
 * on.  The wait gives up after wait_ms (1..2000, else TP_ERR_BAD_SHAPE) and
 * records a timeout, so a following tp_check_device_error() must return
 * TP_ERR_DEVICE_TIMEOUT while the CUDA context stays usable. */
tp_status tp_debug_watchdog(uint32_t wait_ms, void* stream);

/* The tiling the GEMM entry points use on the current device for an output of
 * M rows x N columns in `groups` groups (colwise: one group per shard;
 * rowwise sum: one group), `swiglu` != 0 for tp_colwise_swiglu:
 *   0  CTA pairs (tcgen05 cta_group::2), 256 x 256 tiles (M >= 256)
 *   1  one CTA per tile, 128 x 256 tiles
 *   2  one CTA per tile, 128 x 128 tiles (when that fills the SMs in fewer
 *      rounds of tiles; never for SwiGLU)
 * A pure query (no launch); -1 if a size is < 1 or no CUDA device is usable. */
int tp_gemm_tile_plan(int64_t M, int64_t N, int groups, int swiglu);

/* Synchronises `stream`, then reports (and clears) the device error word that
 * kernels set: TP_ERR_DEVICE_TIMEOUT if a bounded wait ran out, else
 * TP_ERR_RANGE if an epilogue that stores fp16 (the Q/K/V of the attention
 * layers, or tp_colwise_linear with TP_OUT_F16) produced a value whose fp16
 * rounding is +-inf or NaN (|v| >= 65520, or NaN), else TP_OK.  The kernel
 * that sets TP_ERR_RANGE still writes its whole output (the affected values
 * as +-inf or NaN) and the context stays usable; the status says the output
 * of that call must not be trusted.  Returns TP_ERR_CUDA if the
 * synchronisation itself fails. */
tp_status tp_check_device_error(void* stream);

/* ---------------------------------------------------------------------------
 * a1. Shard slicing (style table, "Colwise and rowwise"; "Fused projections").
 * Bit-exact copies; a coalesced 128-bit vectorised HBM copy kernel.
 * ------------------------------------------------------------------------- */

/* out = slice `rank` of W[rows x cols] in `style` (TP_ROWWISE_SPLIT_INPUT
 * slices like TP_ROWWISE).
 *   colwise: out is [rows/T x cols] = W[rank*rows/T : (rank+1)*rows/T, :]
 *   rowwise: out is [rows x cols/T] = W[:, rank*cols/T : (rank+1)*cols/T]
 * Errors: NULL, BAD_STYLE, BAD_DEGREE, BAD_RANK, BAD_SHAPE (rows or cols < 1),
 * INDIVISIBLE (sharded dim % T), ALIGNMENT (pointers, or row lengths of W or
 * out not multiples of 8 elements). */
tp_status tp_shard_weight(const uint16_t* W, int64_t rows, int64_t cols, int style,
                          int tp_degree, int rank, uint16_t* out, void* stream);

/* All T shards of W in one launch, stacked in rank order:
 *   colwise: out is [T x rows/T x cols] (the same bytes as W: a colwise shard
 *            of a row-major weight is a contiguous block of rows);
 *   rowwise: out is [T x rows x cols/T].
 * Same checks as tp_shard_weight (without `rank`). */
tp_status tp_shard_weight_all(const uint16_t* W, int64_t rows, int64_t cols, int style,
                              int tp_degree, uint16_t* out, void* stream);

/* Several all-shard slicing jobs in one launch (e.g. W_up, b_up and W_down of
 * an MLP pair).  jobs[] is HOST memory, 1 <= njobs <= 8 (else BAD_SHAPE).  A
 * job with blocks == NULL is a tp_shard_weight_all job; with blocks != NULL
 * it is a tp_shard_packed_all job (blocks[] in host memory, nblocks of them).
 * Every job is checked as the corresponding single call before anything is
 * launched.  Each job's output is all T shards stacked in rank order.  A
 * colwise layer's bias of n elements is the job {b, T, n/T, TP_COLWISE} (or
 * {b, 1, n, TP_ROWWISE}: the same slices).  One launch for up to 16 plain
 * jobs or packed blocks in all, one more per further 16. */
typedef struct {
  const uint16_t* W;     /* device, [rows x cols] */
  int64_t rows, cols;
  int style;             /* TP_COLWISE, TP_ROWWISE (or TP_ROWWISE_SPLIT_INPUT when plain) */
  uint16_t* out;         /* device, as tp_shard_weight_all's / tp_shard_packed_all's out */
  const int64_t* blocks; /* NULL, or the packed blocks (host) */
  int nblocks;
} tp_shard_job;
tp_status tp_shard_weights_batch(const tp_shard_job* jobs, int njobs, int tp_degree, void* stream);

/* out[n/T] = b[rank*n/T : (rank+1)*n/T] (a colwise layer's bias).  n/T must be
 * a multiple of 8. */
tp_status tp_shard_bias(const uint16_t* b, int64_t n, int tp_degree, int rank,
                        uint16_t* out, void* stream);

/* Head split of a fused QKV weight W_qkv[3D x D] = [Q; K; V] (D rows each,
 * head h at rows h*128 .. h*128+127 inside each block): packed colwise with
 * blocks [1,1,1].  out is [3D/T x D] = [Q_r; K_r; V_r], where X_r holds heads
 * [rank*H/T, (rank+1)*H/T).  Requires D == heads*128 (BAD_SHAPE) and
 * heads % T == 0 (HEADS_INDIVISIBLE). */
tp_status tp_shard_qkv_heads(const uint16_t* W_qkv, int64_t D, int heads, int tp_degree,
                             int rank, uint16_t* out, void* stream);

/* All T head-split shards in one launch: out is [T x 3D/T x D], shard r at
 * out + r*3D/T*D.  Same checks as tp_shard_qkv_heads (without `rank`). */
tp_status tp_shard_qkv_heads_all(const uint16_t* W_qkv, int64_t D, int heads, int tp_degree,
                                 uint16_t* out, void* stream);

/* Packed colwise / rowwise ("Fused projections").  W's packed dimension
 * (dim 0 = rows for TP_COLWISE, dim 1 = cols for TP_ROWWISE) is the
 * concatenation of nblocks blocks.  blocks[] (HOST memory, 1 <= nblocks <= 64)
 * are positive proportional integers whose sum divides the packed dimension
 * P; block b has size S_b = blocks[b] * P / sum (absolute sizes, as stored on
 * a Linear, are the case sum == P).  Each block is sliced on its own and the
 * slices follow one another in block order:
 *   colwise: out is [P/T x cols]: rows [start_b + rank*S_b/T, +S_b/T) of each block;
 *   rowwise: out is [rows x P/T]: those columns of each block.
 * The bias of a packed colwise layer is sliced as a 1 x n matrix with
 * TP_ROWWISE.  Errors, all before any launch: NULL, BAD_STYLE (only
 * TP_COLWISE / TP_ROWWISE), BAD_DEGREE, BAD_RANK, BAD_SHAPE, BAD_BLOCKS,
 * INDIVISIBLE (some S_b % T != 0, even when P % T == 0), ALIGNMENT (cols % 8;
 * rowwise: every S_b/T % 8).  One copy launch per block. */
tp_status tp_shard_packed(const uint16_t* W, int64_t rows, int64_t cols, int style,
                          const int64_t* blocks, int nblocks, int tp_degree, int rank,
                          uint16_t* out, void* stream);

/* All T packed shards, stacked in rank order: out is [T x (shard shape)].
 * Same checks as tp_shard_packed (without `rank`); one launch per block. */
tp_status tp_shard_packed_all(const uint16_t* W, int64_t rows, int64_t cols, int style,
                              const int64_t* blocks, int nblocks, int tp_degree,
                              uint16_t* out, void* stream);

/* ---------------------------------------------------------------------------
 * Step-level calls (each one kernel), on already-sharded operands.
 * ------------------------------------------------------------------------- */

/* a2/a3/a5. Colwise GEMM for every shard:
 *   out[r] = epi( X[M x K] . W_shards[r]^T + b_shards[r] ),   r = 0..T-1
 * W_shards: [T x N_s x K] (shard r's [N_s x K] weight, contiguous);
 * b_shards: [T x N_s] or NULL; out: [T x M x N_s].  epi = GELU(tanh form)
 * when gelu != 0, identity otherwise.  bf16 operands, fp32 accumulation in
 * tensor memory (tcgen05), one rounding at the end to out_dtype
 * (TP_OUT_BF16, or TP_OUT_F16 as used for the Q/K/V that feed attention;
 * anything else is TP_ERR_BAD_STYLE).  With TP_OUT_F16 a value that rounds
 * to +-inf (outside the fp16 range) or is NaN sets the range flag that
 * tp_check_device_error() reports as TP_ERR_RANGE.
 * Requires K % 8 == 0 and N_s % 8 == 0 (ALIGNMENT).  M == 0 is a no-op. */
tp_status tp_colwise_linear(const uint16_t* X, int64_t M, int64_t K,
                            const uint16_t* W_shards, const uint16_t* b_shards, int64_t N_s,
                            int tp_degree, int gelu, int out_dtype, uint16_t* out, void* stream);

/* a4/a7. Rowwise GEMM with the cross-shard sum fused:
 *   Y[M x N] = bf16( sum_r A_shards[r] . W_shards[r]^T + bias )
 * A_shards: [T x M x K_s]; W_shards: [T x N x K_s]; bias: [N] or NULL (added
 * once, after the sum).  One fp32 accumulator walks r = 0..T-1 in order, so
 * no partial is ever written out.  Requires K_s % 8 == 0, N % 8 == 0. */
tp_status tp_rowwise_linear_sum(const uint16_t* A_shards, int64_t M, int64_t K_s,
                                const uint16_t* W_shards, int64_t N, const uint16_t* bias,
                                int tp_degree, uint16_t* Y, void* stream);

/* Row-range forms of the two calls above, for layers whose token sets share
 * one activation buffer (the dual-stream joint attention's Q/K/V and O):
 *   tp_colwise_linear_rows: out is [T x out_rows x N_s] and rows [0, M) of
 *     every shard's block are written (pass out + row_offset*N_s to write
 *     rows [row_offset, row_offset + M)); out_rows >= M (else BAD_SHAPE).
 *   tp_rowwise_linear_sum_rows: A_shards is [T x a_rows x K_s] and rows
 *     [0, M) of every shard's block are read (A_shards + row_offset*K_s for
 *     another range); a_rows >= M (else BAD_SHAPE).
 * Other arguments and checks as tp_colwise_linear / tp_rowwise_linear_sum. */
tp_status tp_colwise_linear_rows(const uint16_t* X, int64_t M, int64_t K,
                                 const uint16_t* W_shards, const uint16_t* b_shards, int64_t N_s,
                                 int tp_degree, int gelu, int out_dtype, uint16_t* out, int64_t out_rows,
                                 void* stream);
tp_status tp_rowwise_linear_sum_rows(const uint16_t* A_shards, int64_t M, int64_t K_s, int64_t a_rows,
                                     const uint16_t* W_shards, int64_t N, const uint16_t* bias,
                                     int tp_degree, uint16_t* Y, void* stream);

/* SwiGLU colwise GEMM for every shard (the gate/up pair packed with blocks
 * [1, 1], section "Fused projections"):
 *   out[r] = silu(X W_gate,r^T + bg_r) * (X W_up,r^T + bu_r),   r = 0..T-1
 * W_shards: [T x 2F_s x K], shard r = [W_gate,r; W_up,r] (F_s rows each: what
 * tp_shard_packed_all(..., TP_COLWISE, {1, 1}, ...) produces); b_shards:
 * [T x 2F_s] = [bg_r, bu_r] per shard, or NULL; out: [T x M x F_s] bf16.
 * silu(x) = x * sigmoid(x).  Both halves accumulate in one tcgen05 tile
 * (gate and up columns side by side in tensor memory) and the product is
 * formed in the epilogue, so neither half is ever written out.
 * Requires K % 8 == 0 and F_s % 8 == 0 (ALIGNMENT).  M == 0 is a no-op. */
tp_status tp_colwise_swiglu(const uint16_t* X, int64_t M, int64_t K,
                            const uint16_t* W_shards, const uint16_t* b_shards, int64_t F_s,
                            int tp_degree, uint16_t* out, void* stream);

/* rowwise_split_input (style table, third row): a rowwise projection whose
 * input is replicated.  Each shard takes its own K/T columns of X:
 *   Y[M x N] = bf16( sum_r X[:, r*K/T : (r+1)*K/T] . W_shards[r]^T + bias )
 * X: [M x K] (the replicated input, read in place: the slice is a TMA
 * coordinate, not a copy); W_shards: [T x N x K/T] (TP_ROWWISE slices of
 * W[N x K]); bias [N] or NULL, added once.  K % T == 0 (INDIVISIBLE);
 * K/T % 8 == 0 and N % 8 == 0 (ALIGNMENT). */
tp_status tp_rowwise_split_input_linear(const uint16_t* X, int64_t M, int64_t K,
                                        const uint16_t* W_shards, int64_t N, const uint16_t* bias,
                                        int tp_degree, uint16_t* Y, void* stream);

/* a6. Per-shard scaled dot-product attention, non-causal, scale 1/sqrt(128):
 * QKV: fp16 [T x M x 3*Hs*128] with Hs = heads/T; inside a row: Q heads,
 * then K heads, then V heads, 128 columns per head (the colwise QKV output,
 * stored in fp16 by the attention block).
 * O: bf16 [T x M x Hs*128], O[r][:, j*128:(j+1)*128] = softmax(Q K^T/sqrt(128)) V
 * for head j of shard r.  Online softmax (running max and sum, fp32), P
 * rounded to fp16 for the P.V product, fp32 accumulation. */
tp_status tp_sdpa_shards(const uint16_t* QKV, int64_t M, int heads, int tp_degree,
                         uint16_t* O, void* stream);

/* a8. Standalone partial-sum reduction (the per-element meaning of the
 * block-boundary AllReduce; the unfused alternative of a4):
 *   Y[M x N] = bf16( sum_{r ascending} parts[r] + bias )
 * parts: fp32 [T x M x N]; bias: [N] bf16 or NULL.  N % 8 == 0. */
tp_status tp_reduce_partials(const float* parts, int64_t M, int64_t N, int tp_degree,
                             const uint16_t* bias, uint16_t* Y, void* stream);

/* ---------------------------------------------------------------------------
 * Layer calls.  The one-shot calls slice the full weights into the caller's
 * workspace (a1) and then run the layer; the prepare/run pair slices once
 * into library-owned memory and runs many times, like sharding at load time
 * and running a forward every step.
 * ------------------------------------------------------------------------- */

/* MLP pair: Y = bf16( sum_r GELU(X W_up,r^T + b_up,r) W_down,r^T + b_down ).
 * X[M x D], W_up[F x D] (colwise), b_up[F], W_down[D x F] (rowwise), b_down[D],
 * Y[M x D].  F % T == 0 (INDIVISIBLE); D and F/T multiples of 8 (ALIGNMENT).
 * b_up / b_down may be NULL (no bias).  Workspace: tp_mlp_workspace_bytes(). */
size_t tp_mlp_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree);
tp_status tp_mlp_pair(const uint16_t* X, int64_t M, int64_t D, int64_t F,
                      const uint16_t* W_up, const uint16_t* b_up,
                      const uint16_t* W_down, const uint16_t* b_down,
                      int tp_degree, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* SwiGLU MLP pair: Y = bf16( sum_r (silu(X W_gate,r^T + bg_r) * (X W_up,r^T + bu_r)) W_out,r^T + b_out ).
 * X[M x D]; W_in[2F x D] = [W_gate; W_up] (packed colwise, blocks [1, 1]);
 * b_in[2F] = [b_gate, b_up] or NULL; W_out[D x F] (rowwise); b_out[D] or
 * NULL; Y[M x D].  F % T == 0 (INDIVISIBLE); D and F/T multiples of 8
 * (ALIGNMENT).  Workspace: tp_swiglu_workspace_bytes(). */
size_t tp_swiglu_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree);
tp_status tp_swiglu_mlp_pair(const uint16_t* X, int64_t M, int64_t D, int64_t F,
                             const uint16_t* W_in, const uint16_t* b_in,
                             const uint16_t* W_out, const uint16_t* b_out,
                             int tp_degree, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* Attention block: Y = bf16( sum_r O_r W_o,r^T ), O_r = per-shard SDPA of the
 * head-split QKV projection X W_qkv,r^T.  X[M x D], W_qkv[3D x D], W_o[D x D],
 * Y[M x D]; D == heads*128; heads % T == 0.  No biases.  Q, K and V are held
 * in fp16: a projection value outside the fp16 range makes the next
 * tp_check_device_error() return TP_ERR_RANGE (the attention weights P are
 * at most 2^8 by construction and cannot overflow).
 * Workspace: tp_attn_workspace_bytes(). */
size_t tp_attn_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree);
tp_status tp_attn_block(const uint16_t* X, int64_t M, int64_t D,
                        const uint16_t* W_qkv, const uint16_t* W_o, int heads, int tp_degree,
                        uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* Load-once / run-many.  *handle receives a library object that owns the
 * sharded weights (device memory allocated here, freed by tp_destroy).  The
 * slicing is enqueued on `stream`; later runs must be ordered after it.
 * tp_*_run_workspace_bytes(M, ...) gives the activation workspace a run needs. */
tp_status tp_mlp_prepare(const uint16_t* W_up, const uint16_t* b_up,
                         const uint16_t* W_down, const uint16_t* b_down,
                         int64_t D, int64_t F, int tp_degree, void* stream, void** handle);
/* The SwiGLU pair's load-once form; arguments as tp_swiglu_mlp_pair.  The
 * handle runs through tp_mlp_run with tp_mlp_run_workspace_bytes. */
tp_status tp_swiglu_prepare(const uint16_t* W_in, const uint16_t* b_in,
                            const uint16_t* W_out, const uint16_t* b_out,
                            int64_t D, int64_t F, int tp_degree, void* stream, void** handle);
size_t tp_mlp_run_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree);
tp_status tp_mlp_run(void* handle, const uint16_t* X, int64_t M, uint16_t* Y,
                     void* ws, size_t ws_bytes, void* stream);

tp_status tp_attn_prepare(const uint16_t* W_qkv, const uint16_t* W_o, int64_t D, int heads,
                          int tp_degree, void* stream, void** handle);
size_t tp_attn_run_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree);
tp_status tp_attn_run(void* handle, const uint16_t* X, int64_t M, uint16_t* Y,
                      void* ws, size_t ws_bytes, void* stream);

/* Dual-stream joint attention (the text stream's add_q/k/v_proj and
 * to_add_out sharded like the image stream's to_q/k/v and to_out):
 *   QKV_r = [X_img W_qkv_img,r^T ; X_txt W_qkv_txt,r^T]   (image rows first)
 *   O_r   = per-head SDPA of QKV_r over all M_img + M_txt tokens
 *   Y_img = bf16( sum_r O_r[:M_img] W_o_img,r^T ),  Y_txt = bf16( sum_r O_r[M_img:] W_o_txt,r^T )
 * X_img[M_img x D], X_txt[M_txt x D]; W_qkv_*[3D x D] = [Q; K; V] (head split
 * as tp_shard_qkv_heads); W_o_*[D x D]; Y_img[M_img x D], Y_txt[M_txt x D].
 * D == heads*128, heads % T == 0, no biases.  Either stream may be empty
 * (its X and Y may then be NULL; M_txt == 0 gives tp_attn_block's result on
 * the image stream).  Both streams' Q/K/V go into one buffer and one SDPA
 * launch; each out-projection reads its stream's rows of O in place.
 * Scheduling: when both streams have tokens, each text-stream projection runs
 * on a stream the library owns (one per device), forked from `stream` and
 * joined back into it with events, beside the image stream's projection on
 * the remaining SMs; the results are the same bits as in sequence, the call
 * can be captured into a CUDA graph, and calls from several host threads are
 * serialized on that internal stream.
 * Workspace: tp_joint_attn_workspace_bytes(). */
size_t tp_joint_attn_workspace_bytes(int64_t M_img, int64_t M_txt, int64_t D, int heads, int tp_degree);
tp_status tp_joint_attn_block(const uint16_t* X_img, int64_t M_img, const uint16_t* X_txt, int64_t M_txt,
                              int64_t D, const uint16_t* W_qkv_img, const uint16_t* W_qkv_txt,
                              const uint16_t* W_o_img, const uint16_t* W_o_txt, int heads, int tp_degree,
                              uint16_t* Y_img, uint16_t* Y_txt, void* ws, size_t ws_bytes, void* stream);
tp_status tp_joint_attn_prepare(const uint16_t* W_qkv_img, const uint16_t* W_qkv_txt,
                                const uint16_t* W_o_img, const uint16_t* W_o_txt, int64_t D, int heads,
                                int tp_degree, void* stream, void** handle);
size_t tp_joint_attn_run_workspace_bytes(int64_t M_img, int64_t M_txt, int64_t D, int heads, int tp_degree);
tp_status tp_joint_attn_run(void* handle, const uint16_t* X_img, int64_t M_img, const uint16_t* X_txt,
                            int64_t M_txt, uint16_t* Y_img, uint16_t* Y_txt, void* ws, size_t ws_bytes,
                            void* stream);

/* ---------------------------------------------------------------------------
 * Context parallelism pieces (page "Context parallelism": Ring attention
 * passes key/value blocks around a ring of ranks, each attending its own
 * queries to the block it holds; Ulysses attention regroups all tokens x a
 * subset of heads onto each rank with an all-to-all, attends locally and
 * regroups back).  These calls are the per-rank compute and layout steps;
 * the exchanges themselves (ring send/recv, all-to-all) are the caller's
 * collectives (NCCL over NVLink); nothing here communicates.
 * ------------------------------------------------------------------------- */

/* One key/value block of Ring attention, for every shard and head:
 *   O[r][i, 128h:128h+128] = softmax_j(Q_i K_j^T / sqrt(128)) V_j   over the block's keys j,
 *   lse[r][h][i] = log2 sum_j 2^(log2(e) Q_i K_j^T / sqrt(128))     (log2 units).
 * Q_qkv: fp16 [T x Mq x 3*Hs*128] (its Q columns are used); KV_qkv: fp16
 * [T x Mk x 3*Hs*128] (its K and V columns; may be the same buffer as Q_qkv,
 * or another rank's block), Hs = heads / T.  O: fp16 [T x Mq x Hs*128], O
 * normalised over this block's keys (a convex combination of fp16 rows of V,
 * so always in fp16 range; rounded once, 2^-11 relative); lse: fp32
 * [T x Hs x Mq].  Mk >= 1.
 * Errors: NULL, BAD_DEGREE, BAD_SHAPE, HEADS_INDIVISIBLE, ALIGNMENT. */
tp_status tp_sdpa_block_stats(const uint16_t* Q_qkv, int64_t Mq, const uint16_t* KV_qkv, int64_t Mk, int heads,
                              int tp_degree, uint16_t* O, float* lse, void* stream);

/* Merge of nparts (1..64) block results into the attention over all their
 * keys: O = sum_b 2^(lse_b - L) O_b / sum_b 2^(lse_b - L), L = max_b lse_b,
 * written in bf16 like tp_sdpa_shards' output; lse_out (or NULL) receives
 * L + log2 sum_b 2^(lse_b - L).  O_parts: fp16 [nparts x T x M x Hs*128]
 * (tp_sdpa_block_stats' output), summed in fp32; lse_parts: fp32
 * [nparts x T x Hs x M]; O: bf16 [T x M x Hs*128]; lse_out: fp32
 * [T x Hs x M]. */
tp_status tp_attn_merge(const uint16_t* O_parts, const float* lse_parts, int nparts, int64_t M, int heads,
                        int tp_degree, uint16_t* O, float* lse_out, void* stream);

/* Inverse of tp_shard_weight_all(..., TP_ROWWISE, ...): src [T x rows x cols/T]
 * (block r) -> out [rows x cols] with block r at columns [r*cols/T, (r+1)*cols/T).
 * Ulysses attention uses the rowwise / packed-rowwise slicing to group each
 * rank's heads by destination before the all-to-all, and this call to put
 * every head group back in place after the reverse all-to-all.  Bit-exact.
 * cols % T == 0 (INDIVISIBLE); cols/T % 8 == 0 (ALIGNMENT). */
tp_status tp_unshard_rowwise_all(const uint16_t* src, int64_t rows, int64_t cols, int tp_degree, uint16_t* out,
                                 void* stream);

/* ---------------------------------------------------------------------------
 * One rank's share of a layer under tensor parallelism ACROSS processes (one
 * process per GPU).  Page "Tensor parallelism", opening paragraph and the
 * paragraph under the "Colwise and rowwise" table: rank r holds only its own
 * shards, the colwise projection's output stays sharded on that rank, and the
 * rowwise projection that follows yields a partial sum; a single AllReduce at
 * the block boundary adds the partials.
 *
 * These calls compute rank r's partial of the layer output in fp32 [M x D],
 * WITHOUT the rowwise bias.  The caller then sums the partials of all ranks
 * with one AllReduce(sum) in fp32 (NCCL over NVLink; nothing here
 * communicates) and finishes on every rank with
 * tp_reduce_partials(summed, M, D, 1, b_down, Y): the bias added once, after
 * the sum, and one bf16 rounding.  Summing the T partials of one process on
 * one GPU with tp_reduce_partials(parts, M, D, T, b_down, Y) gives the same
 * layer.  The rank index is implicit in the shards passed.
 *
 * MLP pair: X [M x D] (replicated); W_up_r [F/T x D] and b_up_r [F/T] (or
 * NULL) = tp_shard_weight / tp_shard_bias of W_up, b_up for this rank;
 * W_down_r [D x F/T] = tp_shard_weight(W_down, TP_ROWWISE, rank);
 * part [M x D] fp32.  Same shape checks as tp_mlp_pair.  Workspace (this
 * rank's hidden activations H_r, bf16): tp_mlp_rank_workspace_bytes().
 *
 * Attention block: X [M x D]; W_qkv_r [3D/T x D] = tp_shard_qkv_heads(W_qkv,
 * ..., rank); W_o_r [D x D/T] = tp_shard_weight(W_o, D, D, TP_ROWWISE, ...,
 * rank); part [M x D] fp32.  Same checks as tp_attn_block (Q/K/V in fp16 with
 * the same TP_ERR_RANGE report).  Workspace: tp_attn_rank_workspace_bytes().
 * ------------------------------------------------------------------------- */
size_t tp_mlp_rank_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree);
tp_status tp_mlp_rank_partial(const uint16_t* X, int64_t M, int64_t D, int64_t F, const uint16_t* W_up_r,
                              const uint16_t* b_up_r, const uint16_t* W_down_r, int tp_degree, float* part, void* ws,
                              size_t ws_bytes, void* stream);
size_t tp_attn_rank_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree);
tp_status tp_attn_rank_partial(const uint16_t* X, int64_t M, int64_t D, const uint16_t* W_qkv_r,
                               const uint16_t* W_o_r, int heads, int tp_degree, float* part, void* ws,
                               size_t ws_bytes, void* stream);

/* Frees a handle from tp_*_prepare (synchronises the device first). NULL is a no-op. */
void tp_destroy(void* handle);

/* ---------------------------------------------------------------------------
 * Allocation-free MLP pair.  The paper has no counterpart: this entry point
 * exists for callers that must not allocate device memory themselves or
 * through the library, e.g. code whose device memory is owned by another
 * allocator (a raw cudaMalloc would bypass its accounting and can fail when
 * that allocator holds most of the device), or code that cannot accept the
 * device-wide synchronisation cudaMalloc/cudaFree may cause.
 *
 * Same result as tp_mlp_pair on already-sharded weights (what each rank holds
 * after sharded loading; tp_shard_weight_all produces them into caller
 * memory without allocating):
 *   W_up_shards [T x F/T x D], b_up_shards [T x F/T] or NULL,
 *   W_down_shards [T x D x F/T], b_down [D] or NULL, X [M x D], Y [M x D].
 * The hidden activations live in a file-scope device array of
 * TP_NOALLOC_SCRATCH_BYTES (64 MiB) that every GPU loading the library holds
 * until the process exits.  Tokens are processed in chunks of
 * floor(64 MiB / (2*F)) rows rounded down to a multiple of 128; if even 128
 * rows do not fit (F > 262144) the call returns TP_ERR_SCRATCH_LIMIT before
 * launching anything.  Other checks as tp_mlp_pair.
 * The first call on a device looks up the array's device address (once per
 * device); make that first call before any stream capture.  Under CUDA's
 * default lazy module loading that first lookup is also when the driver
 * creates the 64 MiB array on that device, so make the first call at start-up,
 * before another allocator takes the device's free memory: after it, calls
 * change the device's free memory by nothing.  Every call shares
 * the one array: calls that overlap on the GPU (different streams, or
 * different host threads on one device) race and corrupt each other's
 * results.  Nothing in the array has to start at zero: a chunk's activations
 * are written in full before they are read, and reads past a chunk's rows
 * come from the TMA unit's out-of-bounds zero fill, never from the array.
 * Calls no cudaMalloc, cudaFree or other allocating routine. */
#define TP_NOALLOC_SCRATCH_BYTES (64ull << 20)
tp_status tp_mlp_pair_sharded_noalloc(const uint16_t* X, int64_t M, int64_t D, int64_t F,
                                      const uint16_t* W_up_shards, const uint16_t* b_up_shards,
                                      const uint16_t* W_down_shards, const uint16_t* b_down,
                                      int tp_degree, uint16_t* Y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TP_B200_TP_H_ */
