// reduce.cu - a8, the standalone partial-sum reduction:
//   Y[M x N] = bf16( sum_{r = 0..T-1} parts[r][M x N] + bias[N] )
// This is what the block-boundary AllReduce computes for each element; the
// fused rowwise GEMM makes it unnecessary on the layer path, and it is kept as
// the unfused alternative.  HBM-bound: each thread owns 8 consecutive columns
// (two 16-byte fp32 loads per shard, one 16-byte bf16 store), shards are summed
// in ascending order in fp32.
#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) reduce_partials_kernel(const float4* __restrict__ parts,
                                                                   const uint16_t* __restrict__ bias,
                                                                   uint4* __restrict__ Y, int64_t n8_total,
                                                                   uint32_t n8_row, int64_t shard_stride4, int T) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n8_total; i += stride) {
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    const float4* p = parts + 2 * i;
    // Issue every shard's loads before the adds (T is small), then sum in order.
    if (T <= 8) {
      float4 lo[8], hi[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < T) {
          lo[r] = __ldcs(p + r * shard_stride4);
          hi[r] = __ldcs(p + r * shard_stride4 + 1);
        }
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < T) {
          acc[0] += lo[r].x; acc[1] += lo[r].y; acc[2] += lo[r].z; acc[3] += lo[r].w;
          acc[4] += hi[r].x; acc[5] += hi[r].y; acc[6] += hi[r].z; acc[7] += hi[r].w;
        }
    } else {
      for (int r = 0; r < T; ++r) {
        const float4 a = __ldcs(p + r * shard_stride4);
        const float4 b = __ldcs(p + r * shard_stride4 + 1);
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
      }
    }
    if (bias != nullptr) {
      const uint32_t c8 = uint32_t(i % n8_row);
      const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bias) + c8);
      acc[0] += bf16_lo(bv.x); acc[1] += bf16_hi(bv.x);
      acc[2] += bf16_lo(bv.y); acc[3] += bf16_hi(bv.y);
      acc[4] += bf16_lo(bv.z); acc[5] += bf16_hi(bv.z);
      acc[6] += bf16_lo(bv.w); acc[7] += bf16_hi(bv.w);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    __stcs(Y + i, o);
  }
}

}  // namespace

cudaError_t launch_reduce_partials(const float* parts, int64_t M, int64_t N, int T, const uint16_t* bias,
                                   uint16_t* Y, cudaStream_t s) {
  const int64_t n8_total = M * N / 8;
  if (n8_total == 0) return cudaSuccess;
  int64_t blocks = (n8_total + kThreads - 1) / kThreads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  reduce_partials_kernel<<<unsigned(blocks), kThreads, 0, s>>>(reinterpret_cast<const float4*>(parts), bias,
                                                               reinterpret_cast<uint4*>(Y), n8_total,
                                                               uint32_t(N / 8), M * N / 4, T);
  count_launch();
  return note_cuda_error("reduce: launch", cudaGetLastError());
}

}  // namespace tp
