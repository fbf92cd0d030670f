// merge.cu - combines per-key-block attention results (Ring attention,
// Diffusers "Context parallelism" page, section on Ring attention: each rank
// attends its queries to the key/value block it holds while the blocks travel
// around the ring, and the partial results are combined).
//
// Block b gives, for one (shard, query row, head), O_b = softmax over its
// keys applied to its values (normalised, fp16) and lse_b = log2 of the sum of
// 2^(scaled score) over its keys.  Over all blocks,
//   O = sum_b 2^(lse_b - L) O_b / sum_b 2^(lse_b - L),   L = max_b lse_b,
// which is exactly softmax over all keys applied to all values (each O_b is
// its block's weighted mean; 2^(lse_b) is its block's total weight).
// HBM-bound: a thread owns 8 consecutive columns of one row and head (one
// 16-byte fp16 load per block, one 16-byte bf16 store); for up to 8 blocks
// all of a group's loads are in flight before the sum, which is fp32.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

constexpr int kThreads = 256;

// Index of column group i's row statistics: groups run over (t, row, head,
// 8-column chunk) with 16 chunks per head.
__device__ __forceinline__ int64_t lse_index(int64_t i, int64_t M, int Hs) {
  const int64_t row_groups = int64_t(Hs) * 16;  // 8-column groups per row
  const int64_t tr = i / row_groups;            // t * M + row
  const int head = int(i - tr * row_groups) >> 4;
  const int64_t t = tr / M, row = tr - t * M;
  return (t * Hs + head) * M + row;
}

// acc += w * (8 fp16 values of one block), in fp32
__device__ __forceinline__ void add_block(float (&acc)[8], float w, const uint4& v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
    acc[2 * k] += w * f.x;
    acc[2 * k + 1] += w * f.y;
  }
}

// Writes group i's merged values (bf16) and, for its first group of a
// head, the merged log-sum-exp.
__device__ __forceinline__ void write_group(int64_t i, int64_t li, const float (&acc)[8], float wsum, float L,
                                            uint4* __restrict__ O, float* __restrict__ lse_out) {
  const float inv = 1.0f / wsum;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  __stcs(O + i, o);
  if (lse_out != nullptr && (i & 15) == 0) lse_out[li] = L + log2f(wsum);
}

// kNP > 0: the block count is a compile-time constant, so all kNP loads of a
// column group are issued before its weighted sum (all in flight at once);
// kNP == 0 walks a run-time count one block at a time.  Both sum the blocks in
// ascending order.
template <int kNP>
__global__ void __launch_bounds__(kThreads)
    attn_merge_kernel(const uint4* __restrict__ O_parts, const float* __restrict__ lse_parts, int nparts, int64_t M,
                      int Hs, int64_t n8_total, uint4* __restrict__ O, float* __restrict__ lse_out) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  const int64_t part_stride = n8_total;      // 16-byte groups (8 fp16) per block's O
  const int64_t lse_stride = n8_total / 16;  // T * Hs * M values per block
  const int64_t first = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  if constexpr (kNP > 0) {
    for (int64_t i = first; i < n8_total; i += stride) {
      const int64_t li = lse_index(i, M, Hs);
      float lse[kNP];
      uint4 v[kNP];
#pragma unroll
      for (int b = 0; b < kNP; ++b) {
        lse[b] = lse_parts[b * lse_stride + li];
        v[b] = __ldcs(O_parts + b * part_stride + i);
      }
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float wsum = 0.f, L = -INFINITY;
#pragma unroll
      for (int b = 0; b < kNP; ++b) L = fmaxf(L, lse[b]);
#pragma unroll
      for (int b = 0; b < kNP; ++b) {
        const float w = exp2f(lse[b] - L);
        wsum += w;
        add_block(acc, w, v[b]);
      }
      write_group(i, li, acc, wsum, L, O, lse_out);
    }
  } else {
    for (int64_t i = first; i < n8_total; i += stride) {
      const int64_t li = lse_index(i, M, Hs);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float wsum = 0.f, L = -INFINITY;
      for (int b = 0; b < nparts; ++b) L = fmaxf(L, lse_parts[b * lse_stride + li]);
      for (int b = 0; b < nparts; ++b) {
        const float w = exp2f(lse_parts[b * lse_stride + li] - L);
        wsum += w;
        add_block(acc, w, __ldcs(O_parts + b * part_stride + i));
      }
      write_group(i, li, acc, wsum, L, O, lse_out);
    }
  }
}

}  // namespace

cudaError_t launch_attn_merge(const uint16_t* O_parts, const float* lse_parts, int nparts, int64_t M, int Hs, int T,
                              uint16_t* O, float* lse_out, cudaStream_t s) {
  const int64_t n8_total = int64_t(T) * M * Hs * 16;
  if (n8_total == 0) return cudaSuccess;
  int64_t blocks = (n8_total + kThreads - 1) / kThreads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  using Kernel = void (*)(const uint4*, const float*, int, int64_t, int, int64_t, uint4*, float*);
  constexpr Kernel by_count[9] = {attn_merge_kernel<0>, attn_merge_kernel<1>, attn_merge_kernel<2>,
                                  attn_merge_kernel<3>, attn_merge_kernel<4>, attn_merge_kernel<5>,
                                  attn_merge_kernel<6>, attn_merge_kernel<7>, attn_merge_kernel<8>};
  const Kernel kernel = nparts <= 8 ? by_count[nparts] : attn_merge_kernel<0>;
  kernel<<<unsigned(blocks), kThreads, 0, s>>>(reinterpret_cast<const uint4*>(O_parts), lse_parts, nparts, M, Hs,
                                               n8_total, reinterpret_cast<uint4*>(O), lse_out);
  count_launch();
  return note_cuda_error("attention merge: launch", cudaGetLastError());
}

}  // namespace tp
