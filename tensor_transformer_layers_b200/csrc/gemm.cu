// gemm.cu - the colwise and rowwise projections of a TP layer pair on the
// 5th-generation tensor cores (tcgen05), fed by TMA, accumulating in tensor
// memory (TMEM).
//
// One kernel serves both styles of the Diffusers "Tensor parallelism" page
// (section "Colwise and rowwise", style table):
//   colwise  out_r = epi(X . W_r^T + b_r) for every shard r: the tile's K loop
//            covers the shared input X against shard r's weight rows;
//   rowwise  Y = sum_r A_r . W_r^T + b: the tile's K loop walks every shard's
//            K range in ascending r into ONE fp32 accumulator, so the sum the
//            block-boundary AllReduce performs happens inside the accumulator
//            and the bias is added once in the epilogue.
//
// Structure (one CTA per SM, persistent over output tiles, 192 threads):
//   warp 0   TMA producer: 128x64 A tile + 256x64 B tile per stage, 128-byte
//            swizzle, 4-stage ring of full/empty mbarriers.
//   warp 1   TMEM allocator + MMA issuer: one thread issues 4 x
//            tcgen05.mma (M=128, N=256, K=16) per stage, commits the stage
//            back to the producer, and commits a finished accumulator to the
//            epilogue.  Two 256-column fp32 accumulators (all 512 TMEM
//            columns) let tile i+1's MMAs run while tile i drains.
//   warps 2-5 epilogue: tcgen05.ld 32 columns at a time (thread = output
//            row), bias, optional tanh-form GELU, rounding to bf16 (or fp16
//            for the Q/K/V projection that feeds attention), 16-byte global
//            stores; then release the accumulator.
// Every mbarrier wait is bounded (see ptx.cuh): a wait that runs out sets the
// device error word, the CTA's roles stop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the kernel returns.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;
constexpr int kBBytes = BN * BK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccCols = BN;      // fp32 TMEM columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers + 1 KB alignment slack
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN, false);

static_assert(kTmemCols == 512, "two 256-column accumulators fill TMEM");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ float gelu_tanh(float x) {
  // 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))  (Hendrycks & Gimpel, 2016)
  const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return 0.5f * x * (1.0f + tanh_approx(u));
}

struct TileCoord {
  int g, mb, nb;
};

__device__ __forceinline__ TileCoord decode_tile(int t, int m_tiles, int n_tiles) {
  const int per = m_tiles * n_tiles;
  TileCoord c;
  c.g = t / per;
  const int rem = t - c.g * per;
  c.mb = rem / n_tiles;
  c.nb = rem - c.mb * n_tiles;
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                   const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (p.M + BM - 1) / BM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int tiles = m_tiles * n_tiles * p.groups;
  const int k_iters = p.k_blocks * p.kshards;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile(t, m_tiles, n_tiles);
        for (int it = 0; it < k_iters; ++it) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int s = it / p.k_blocks;
          const int kb = it - s * p.k_blocks;
          uint8_t* sa = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_3d(sa, &amap, &full[stage], kb * BK, tc.mb * BM, p.a_follows_shard ? s : 0);
          tma_load_3d(sa + kABytes, &bmap, &full[stage], kb * BK, tc.nb * BN, tc.g + s);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        // Let every issued copy land before the CTA's shared memory goes away.
        // Stage s was last armed in the current phase if s < stage, else in the previous one.
        const volatile int no_abort = 0;
        for (int s = 0; s < kStages; ++s) {
          if (issued <= s) break;
          mbar_wait(&full[s], s < stage ? phase : (phase ^ 1u), &no_abort);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
        const int acc = local & 1;
        if (!mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * kAccCols);
        for (int it = 0; it < k_iters; ++it) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint64_t da = sdesc_sw128(sa, 16, 1024);
          const uint64_t db = sdesc_sw128(sa + kABytes, 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // advance 16 bf16 = 32 bytes inside the swizzle row
            umma_ss(d_tmem, da + uint64_t(2 * k), db + uint64_t(2 * k), kIdesc, (it | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        // Wait for every MMA already issued before TMEM is released.
        const volatile int no_abort = 0;
        umma_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // this warp's TMEM lane quarter
    int local = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const TileCoord tc = decode_tile(t, m_tiles, n_tiles);
      const int acc = local & 1;
      if (!mbar_wait(&tfull[acc], (local >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row = tc.mb * BM + q * 32 + lane;
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kAccCols);
      uint16_t* orow = p.out + int64_t(tc.g) * p.out_gstride + int64_t(row) * p.ldo;
      const uint16_t* bias = p.bias ? p.bias + int64_t(tc.g) * p.bias_gstride : nullptr;
      const int col_base = tc.nb * BN;
      const int n_left = p.N - col_base;
      const int chunks = n_left >= BN ? BN / 32 : (n_left + 31) / 32;  // warp-uniform
      for (int c = 0; c < chunks; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32_sync(taddr + uint32_t(c * 32), r);
        const int col0 = col_base + c * 32;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (bias != nullptr) {
          const uint4* bp = reinterpret_cast<const uint4*>(bias + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (col0 + 8 * j < p.N) {
              const uint4 b = __ldg(bp + j);
              v[8 * j + 0] += bf16_lo(b.x);
              v[8 * j + 1] += bf16_hi(b.x);
              v[8 * j + 2] += bf16_lo(b.y);
              v[8 * j + 3] += bf16_hi(b.y);
              v[8 * j + 4] += bf16_lo(b.z);
              v[8 * j + 5] += bf16_hi(b.z);
              v[8 * j + 6] += bf16_lo(b.w);
              v[8 * j + 7] += bf16_hi(b.w);
            }
          }
        }
        if (p.gelu) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
        }
        uint4 o[4];
        if (p.out_f16) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            o[j].x = pack_f16x2(v[8 * j + 0], v[8 * j + 1]);
            o[j].y = pack_f16x2(v[8 * j + 2], v[8 * j + 3]);
            o[j].z = pack_f16x2(v[8 * j + 4], v[8 * j + 5]);
            o[j].w = pack_f16x2(v[8 * j + 6], v[8 * j + 7]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            o[j].x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
            o[j].y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
            o[j].z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
            o[j].w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
          }
        }
        if (row < p.M) {
          uint4* op = reinterpret_cast<uint4*>(orow + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (col0 + 8 * j < p.N) op[j] = o[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (!ok && lane == 0) report_timeout(p.err, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& amap, const CUtensorMap& bmap, const GemmArgs& a, int num_sms,
                        cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.groups <= 0) return cudaSuccess;
  const int m_tiles = (a.M + BM - 1) / BM;
  const int n_tiles = (a.N + BN - 1) / BN;
  const int64_t tiles = int64_t(m_tiles) * n_tiles * a.groups;
  const int grid = int(tiles < num_sms ? tiles : num_sms);
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(amap, bmap, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tp
