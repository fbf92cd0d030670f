// internal.h - launchers shared between the C-ABI layer (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace tp {

// ----------------------------------------------------------------------------
// a1: blocked 2-D copy.  For b in [0, nblocks), b2 in [0, nblocks2),
// r in [0, rows), c in [0, cols):
//   dst[b*dst_bstride + b2*dst_bstride2 + r*dst_ld + c]
//     = src[b*src_bstride + b2*src_bstride2 + r*src_ld + c]
// (element units; dst_ld < 0 means dst_ld = cols).  cols, src_ld, dst_ld, the
// strides and both pointers must be multiples of 8 elements / 16 bytes
// (checked by the caller).
// ----------------------------------------------------------------------------
cudaError_t launch_slice_copy(const uint16_t* src, uint16_t* dst, int64_t nblocks, int64_t rows, int64_t cols,
                              int64_t src_ld, int64_t src_bstride, int64_t dst_bstride, cudaStream_t s,
                              int64_t nblocks2 = 1, int64_t src_bstride2 = 0, int64_t dst_bstride2 = 0,
                              int64_t dst_ld = -1);

// Blocked 2-D copies (same meaning as above, one block index), up to
// kSliceJobsPerLaunch in one launch.  Element units; cols, the lds, the
// strides and both pointers multiples of 8 elements / 16 bytes.
// kMaxSliceJobs bounds the jobs of one tp_shard_weights_batch call (each may
// expand into several copies: one per packed block).
constexpr int kMaxSliceJobs = 8;
constexpr int kSliceJobsPerLaunch = 16;
struct SliceJob {
  const uint16_t* src;
  uint16_t* dst;
  int64_t nblocks, rows, cols, src_ld, dst_ld, src_bstride, dst_bstride;
};
cudaError_t launch_slice_jobs(const SliceJob* jobs, int njobs, cudaStream_t s);

// ----------------------------------------------------------------------------
// a8: Y[M x N] = bf16(sum_r parts[r] + bias)
// ----------------------------------------------------------------------------
cudaError_t launch_reduce_partials(const float* parts, int64_t M, int64_t N, int T, const uint16_t* bias,
                                   uint16_t* Y, cudaStream_t s);

// ----------------------------------------------------------------------------
// GEMM (tcgen05).  Computes, for each output group g and tile:
//   out_g[M x N] = epi( sum_{s in K-shards of g} A_{za(s)} . B_{zb(g,s)}^T + bias_g )
// A map: 3-D bf16 {K_s, M, ZA}; B map: 3-D bf16 {K_s, Nrows, ZB}.
//   colwise: groups = T, kshards = 1, zb = g, za = 0.
//   rowwise: groups = 1, kshards = T, zb = s, za = s.
//   rowwise_split_input: as rowwise, but A is one replicated [M x T*K_s]
//     input and shard s reads its columns [s*K_s, (s+1)*K_s): the A map is
//     built {K_s, T, M} (a_split_input = 1) and loaded at (k, s, row).
//   SwiGLU colwise (swiglu = 1): B_g = [gate_g; up_g] with up_g starting
//     up_off rows in; each 256-column accumulator holds 128 gate and the 128
//     matching up columns, and the epilogue writes silu(gate + bg) * (up + bu)
//     to a 128-column output tile (N = output columns = gate rows).
// ----------------------------------------------------------------------------
struct GemmArgs {
  int M;                 // output rows
  int N;                 // output columns per group
  int k_blocks;          // ceil(K_s / 64) per shard
  int kshards;           // shards walked by one tile's K loop
  int groups;            // output groups (colwise shards)
  int a_follows_shard;   // 1: A's z coordinate = K-loop shard; 0: z = 0
  void* out;             // bf16 / fp16 / fp32 output
  int64_t out_gstride;   // elements between groups
  int64_t ldo;           // output row stride (elements)
  const uint16_t* bias;  // bf16 bias or nullptr
  int64_t bias_gstride;  // elements between groups' biases
  int gelu;              // 1: tanh-form GELU after bias
  int out_f16;           // 1: store fp16 instead of bf16
  int out_f32;           // 1: store the fp32 accumulator values (after bias / GELU) unrounded
  int swiglu;            // 1: SwiGLU epilogue over [gate; up] weight rows (see above)
  int a_split_input;     // 1: A map is {K_s, T, M}, loaded at (k, s, row)
  int64_t up_off;        // SwiGLU: rows from gate_g to up_g in B (and bias elements)
  int* err;              // device error word
};

// A bf16 operand seen as a 3-D tensor {k (contiguous), rows, z}: the GEMM
// builds its TMA maps from this (box sizes depend on the kernel it picks).
// z-slices lie zrows rows apart in memory (0: zrows = rows), so an operand
// can be a row range of a taller [z][zrows][k] buffer; rows past `rows` read
// as zeros.  With a_split_input the A operand's memory is [rows][z][k] instead.
struct GemmOperand {
  const void* base;
  uint64_t k, rows, z;
  uint64_t zrows = 0;
};

cudaError_t launch_gemm(const GemmOperand& A, const GemmOperand& B, const GemmArgs& a, int num_sms, cudaStream_t s);

// The tiling launch_gemm picks for M output rows x N columns x groups: CTA
// pairs with 256 x 256 tiles, or one CTA per tile with 128 x 256 or 128 x 128
// tiles (the last when it fills the SMs in fewer rounds; never for SwiGLU).
enum { kPlanPair = 0, kPlanCta128x256 = 1, kPlanCta128x128 = 2 };
int gemm_tile_plan(int64_t M, int64_t N, int groups, bool swiglu, int num_sms);  // plan.cu
// CTA pairs of the pair kernel that fit on the current device at once (cached).
int gemm_max_active_pairs(int num_sms);

// ----------------------------------------------------------------------------
// a6: per-shard SDPA (attn.cu).  Queries come from the Q columns of one fp16
// buffer [T][Mq][*], keys and values from the K and V columns of another (or
// the same) buffer [T][Mk][*]; head h of a shard uses columns q_col0 + 128 h,
// k_col0 + 128 h and v_col0 + 128 h.  Maps (fp16, 3-D {columns, rows, T},
// box 64 x 128, 128-byte swizzle): q over the query buffer, kv over the key /
// value buffer; o: the output map over [T][Mq][Hs*128] (bf16 box 64 x 32, or
// fp32 box 32 x 32 in the statistics mode).
// ----------------------------------------------------------------------------
struct AttnMaps {
  CUtensorMap q, kv, o;
};
struct AttnArgs {
  int Mq, Mk;        // query rows, key rows
  int Hs, T;         // heads per shard, shards
  int q_col0, k_col0, v_col0;
  int stats;         // 0: O / l in bf16; 1: O / l in fp32 and lse
  float* lse;        // statistics mode: [T][Hs][Mq] fp32, log2 units (m + log2 l of the scaled scores)
  float scale_log2;  // log2(e)/sqrt(128)
  int* err;
};
cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& a, int num_sms, cudaStream_t s);

// Merge of per-key-block attention results (Ring attention): for every
// (shard, row, head), O = sum_b 2^(lse_b - L) O_b / sum_b 2^(lse_b - L) with
// L = max_b lse_b, written in bf16; lse_out (optional) = L + log2 sum_b
// 2^(lse_b - L).  O_parts [nparts][T][M][Hs*128] fp16, lse_parts
// [nparts][T][Hs][M] fp32 (log2 units), O [T][M][Hs*128] bf16.
cudaError_t launch_attn_merge(const uint16_t* O_parts, const float* lse_parts, int nparts, int64_t M, int Hs, int T,
                              uint16_t* O, float* lse_out, cudaStream_t s);

// One CTA whose bounded wait on an mbarrier that nothing arrives on must run
// out after limit_ns and set kErrTimeout in *err (watchdog.cu).
cudaError_t launch_watchdog_probe(int* err, uint64_t limit_ns, cudaStream_t s);

// Counts kernel launches (api.cu); every launcher calls it once per launch.
void count_launch();

// Shape checks of an MLP pair (M tokens, hidden D, FFN width F, degree T), as
// every MLP entry point applies them (api.cu); returns a tp_status value.
int mlp_shape_status(int64_t M, int64_t D, int64_t F, int T);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Records why a CUDA call failed (thread-local; read by tp_last_error_message)
// and returns `e` so launchers can `return note_cuda_error(...)`.
cudaError_t note_cuda_error(const char* where, cudaError_t e, const char* detail = nullptr);

// SM count and device error word of the current device, initialising the
// library's per-device state (tensor-map encoder included) on first use.
// Returns a tp_status value.
int current_device_context(int* num_sms, int** err);

// Host helpers (api.cu).  d1_stride: elements of dim 1 between dim-2 slices
// (0 = d1, the packed layout).
CUresult make_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                          uint32_t box0, uint32_t box1, uint64_t d1_stride = 0);
CUresult make_map_3d_bf16_box(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t box0, uint32_t box1, uint32_t box2);
// Output map of the GEMM epilogue's TMA stores: 16-bit {n, m, g} with the
// given row and group strides (elements), box 64 x 32, 128-byte swizzle.
CUresult make_map_out_u16(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t g, uint64_t row_stride,
                          uint64_t group_stride);
// The same for fp32 outputs: box 32 x 32 (128-byte rows), 128-byte swizzle.
CUresult make_map_out_f32(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t g, uint64_t row_stride,
                          uint64_t group_stride);
CUresult make_map_3d_f16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                         uint32_t box1);

}  // namespace tp
