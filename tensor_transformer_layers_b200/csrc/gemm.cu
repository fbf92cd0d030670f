// gemm.cu - the colwise and rowwise projections of a TP layer pair on the
// 5th-generation tensor cores (tcgen05), fed by TMA, accumulating in tensor
// memory (TMEM).
//
// One kernel family serves both styles of the Diffusers "Tensor parallelism"
// page (section "Colwise and rowwise", style table):
//   colwise  out_r = epi(X . W_r^T + b_r) for every shard r: the tile's K loop
//            covers the shared input X against shard r's weight rows;
//   rowwise  Y = sum_r A_r . W_r^T + b: the tile's K loop walks every shard's
//            K range in ascending r into ONE fp32 accumulator, so the sum the
//            block-boundary AllReduce performs happens inside the accumulator
//            and the bias is added once in the epilogue.
//
// Two kernels, same roles (192 threads, persistent over output tiles):
//   warp 0    TMA producer (128-byte swizzle, ring of full/empty mbarriers);
//   warp 1    TMEM allocator + single-thread MMA issuer; two 256-column fp32
//             accumulators (all 512 TMEM columns) so tile i's epilogue runs
//             while tile i+1's MMAs do;
//   warps 2-5 epilogue: tcgen05.ld 32 columns at a time (thread = output row),
//             bias, optional tanh-form GELU, rounding to bf16 (or fp16 for the
//             Q/K/V that feed attention); each warp stages its 32 rows x 64
//             columns in shared memory (128-byte swizzle, two buffers) and
//             writes them with one TMA store, so global writes are whole lines
//             instead of 16 bytes from each of 32 rows per instruction; TMA
//             clips the ragged edges.
// Two more forms of the same kernels:
//   SwiGLU colwise (a gate/up pair packed with blocks [1, 1], section "Fused
//            projections"): the B tile's first 128 rows are gate rows and its
//            last 128 the matching up rows, fetched from the two blocks of the
//            shard [gate_r; up_r] as they lie; the epilogue pairs accumulator
//            column j with column 128 + j and writes silu(g) * u, so the output
//            tile is 128 columns wide;
//   rowwise_split_input (style table): A is the replicated input and shard s
//            reads its own K range of it; the A map is {K_s, T, M}, so the
//            slice of the input is a TMA coordinate, not a copy.
// * gemm_tc_kernel<BN>: one CTA per tile, 128xBN tiles, M=128 N=BN K=16
//   MMAs; BN = 256 with 4 stages of 48 KB (A 128x64 + B 256x64), BN = 128 with
//   6 stages of 32 KB.  The host plan (plan.cu) picks it for M < 256 and for
//   problems whose 128x128 tiles fill the SMs in fewer rounds than pairs do.
// * gemm_pair_kernel: CTA pairs (cluster of 2, tcgen05 cta_group::2), 256x256
//   tile per pair.  Each CTA loads its 128 rows of A and its 128 rows of B
//   (32 KB per k-block instead of 48 KB: the B tile is split between the two
//   SMs), so the shared-memory fill per MMA cycle drops by a third and 6
//   stages fit.  The even CTA issues M=256 N=256 K=16 MMAs over both CTAs'
//   shared memory; each CTA's TMEM holds its 128 accumulator rows.  No TMA
//   multicast: each CTA fetches its own tiles.
// Every mbarrier wait is bounded (see ptx.cuh): a wait that runs out sets the
// device error word, the CTA's roles stop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the kernel returns.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kAccCols = 256;  // fp32 TMEM columns per accumulator (N = 256)
constexpr int kTmemCols = 2 * kAccCols;

// epilogue staging: per epilogue warp two buffers of 32 rows x 128 bytes
constexpr int kEpiBuf = 32 * 128;
constexpr int kEpiBytes = 4 * 2 * kEpiBuf;

// single-CTA kernels: 128 x BN tiles, BN = 256 (4 stages) or 128 (6 stages)
constexpr int BM1 = 128;
constexpr int kABytes1 = BM1 * BK * 2;
template <int BN>
struct Cta1 {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kStageBytes = kABytes1 + BN * BK * 2;
  static constexpr int kEpiOff = kStages * kStageBytes;
  static constexpr int kBarOff = kEpiOff + kEpiBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers + 1 KB alignment slack
  static constexpr uint32_t kIdesc = idesc_bf16_f32(BM1, BN, false);
};

// CTA-pair kernel (per CTA: 128 rows of A and 128 rows of B per stage)
constexpr int BM2 = 256, BN2 = 256;
constexpr int kStages2 = 6;
constexpr int kHalfBytes = 128 * BK * 2;
constexpr int kStageBytes2 = 2 * kHalfBytes;
constexpr int kEpiOff2 = kStages2 * kStageBytes2;
constexpr int kBarOff2 = kEpiOff2 + kEpiBytes;
constexpr int kSmemBytes2 = kBarOff2 + 512 + 1024;
constexpr uint32_t kIdesc2 = idesc_bf16_f32(BM2, BN2, false);

static_assert(kTmemCols == 512, "two 256-column accumulators fill TMEM");
static_assert(Cta1<256>::kSmemBytes <= 227 * 1024 && Cta1<128>::kSmemBytes <= 227 * 1024 &&
                  kSmemBytes2 <= 227 * 1024,
              "shared memory budget");

// GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
// (Hendrycks & Gimpel, 2016), on two values at once: the polynomial and the
// final product in packed fp32 pairs (half the FMA-pipe instructions of the
// scalar form; the epilogue's arithmetic competes with the MMA issue for the
// sub-partitions while the next tile's MMAs run), tanh on the MUFU unit.
__device__ __forceinline__ void gelu_tanh2(float& a, float& b) {
  const uint64_t x = f32x2(a, b);
  const uint64_t x2 = mul_f32x2(x, x);
  const uint64_t inner = fma_f32x2(mul_f32x2(x2, f32x2(0.044715f, 0.044715f)), x, x);  // x + 0.044715 x^3
  float u0, u1;
  f32x2_split(mul_f32x2(inner, f32x2(0.7978845608028654f, 0.7978845608028654f)), u0, u1);
  const uint64_t th = f32x2(tanh_approx(u0), tanh_approx(u1));
  const uint64_t hx = mul_f32x2(x, f32x2(0.5f, 0.5f));
  f32x2_split(fma_f32x2(hx, th, hx), a, b);  // 0.5 x + 0.5 x tanh(u)
}

// SiLU(x) = x * sigmoid(x) = x / (1 + 2^(-x log2 e))  (Elfwing et al., 2018).
// For x -> -inf the power overflows to +inf and the reciprocal to 0.
__device__ __forceinline__ float silu(float x) {
  return x * rcp_approx(1.0f + ex2_approx(-1.4426950408889634f * x));
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

// Stages 16 output bytes (8 columns) of this thread's row at 16-byte chunk k
// (0..7) of a 32-row x 128-byte box in the 128-byte swizzle that the output
// map's TMA store expects (chunk index XOR row index mod 8).
__device__ __forceinline__ void stage16(uint8_t* buf, int lane, int k, uint4 v) {
  *reinterpret_cast<uint4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) = v;
}

// Hands a staged 32 x 64 box to the TMA unit.  `row0` is the warp's first
// row; a box wholly below M is skipped (TMA would clip it anyway).
__device__ __forceinline__ void store_box(const CUtensorMap* omap, uint8_t* buf, int lane, int col0, int row0, int g,
                                          int M) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && row0 < M) {
    tma_store_3d(omap, buf, col0, row0, g);
    bulk_commit();
  }
}

// Waits until the staging buffer about to be reused is no longer read by an
// earlier TMA store of this warp (two buffers, so one store may stay in flight).
__device__ __forceinline__ uint8_t* next_buf(uint8_t* stage, uint32_t& nbox, int lane) {
  uint8_t* buf = stage + (nbox & 1u) * kEpiBuf;
  ++nbox;
  if (lane == 0) bulk_wait_read_1();
  __syncwarp();
  return buf;
}

// fp32 output (a rank's partial sum before the cross-rank AllReduce): each
// 64-column chunk goes out as two 32-row x 32-column fp32 boxes (128-byte rows
// in the output map's 128-byte swizzle); a half wholly past N is skipped.
__device__ __forceinline__ void epilogue_rows_f32(const GemmArgs& p, const CUtensorMap* omap, uint32_t taddr,
                                                  int row0, int lane, int g, int col_base, int width, uint8_t* stage,
                                                  uint32_t& nbox) {
  const uint16_t* bias = p.bias ? p.bias + int64_t(g) * p.bias_gstride : nullptr;
  const int n_left = p.N - col_base;
  const int halves = n_left >= width ? width / 32 : (n_left > 0 ? (n_left + 31) / 32 : 0);  // warp-uniform
  for (int h = 0; h < halves; ++h) {
    uint8_t* buf = next_buf(stage, nbox, lane);
    uint32_t r[32];
    __syncwarp();
    tmem_ld32_sync(taddr + uint32_t(h * 32), r);
    const int col0 = col_base + h * 32;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    if (bias != nullptr) {
      const uint4* bp = reinterpret_cast<const uint4*>(bias + col0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (col0 + 8 * j < p.N) {
          const uint4 bb = __ldg(bp + j);
          const uint32_t w[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            f32x2_split(add_f32x2(f32x2(v[8 * j + 2 * q], v[8 * j + 2 * q + 1]), f32x2(bf16_lo(w[q]), bf16_hi(w[q]))),
                        v[8 * j + 2 * q], v[8 * j + 2 * q + 1]);
        }
      }
    }
    if (p.gelu) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) gelu_tanh2(v[j], v[j + 1]);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      stage16(buf, lane, j,
              make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]), __float_as_uint(v[4 * j + 2]),
                         __float_as_uint(v[4 * j + 3])));
    store_box(omap, buf, lane, col0, row0, g, p.M);
  }
}

// Drains `width` columns of a 128-row fp32 accumulator (this warp's 32 lanes,
// TMEM columns from taddr, output columns from col_base, rows from row0) in
// 64-column boxes: bias, GELU, rounding, staging, TMA store.
__device__ __forceinline__ void epilogue_rows(const GemmArgs& p, const CUtensorMap* omap, uint32_t taddr, int row0,
                                              int lane, int g, int col_base, int width, uint8_t* stage,
                                              uint32_t& nbox) {
  const uint16_t* bias = p.bias ? p.bias + int64_t(g) * p.bias_gstride : nullptr;
  const int n_left = p.N - col_base;
  const int boxes = n_left >= width ? width / 64 : (n_left > 0 ? (n_left + 63) / 64 : 0);  // warp-uniform
  uint32_t nonfinite = 0;  // fp16 outputs: any half that rounded to +-inf or NaN
  for (int b = 0; b < boxes; ++b) {
    uint8_t* buf = next_buf(stage, nbox, lane);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t r[32];
      __syncwarp();
      tmem_ld32_sync(taddr + uint32_t(b * 64 + h * 32), r);
      const int col0 = col_base + b * 64 + h * 32;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      if (bias != nullptr) {
        const uint4* bp = reinterpret_cast<const uint4*>(bias + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (col0 + 8 * j < p.N) {
            const uint4 bb = __ldg(bp + j);
            const uint32_t w[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
              f32x2_split(add_f32x2(f32x2(v[8 * j + 2 * h], v[8 * j + 2 * h + 1]), f32x2(bf16_lo(w[h]), bf16_hi(w[h]))),
                          v[8 * j + 2 * h], v[8 * j + 2 * h + 1]);
          }
        }
      }
      if (p.gelu) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) gelu_tanh2(v[j], v[j + 1]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 o;
        if (p.out_f16) {
          o.x = pack_f16x2(v[8 * j + 0], v[8 * j + 1]);
          o.y = pack_f16x2(v[8 * j + 2], v[8 * j + 3]);
          o.z = pack_f16x2(v[8 * j + 4], v[8 * j + 5]);
          o.w = pack_f16x2(v[8 * j + 6], v[8 * j + 7]);
          // Columns past N are never stored; only the stored ones may raise the flag.
          if (col0 + 8 * j < p.N)
            nonfinite |= f16x2_nonfinite(o.x) | f16x2_nonfinite(o.y) | f16x2_nonfinite(o.z) | f16x2_nonfinite(o.w);
        } else {
          o.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
          o.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
          o.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
          o.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
        }
        stage16(buf, lane, h * 4 + j, o);
      }
    }
    store_box(omap, buf, lane, col_base + b * 64, row0, g, p.M);
  }
  // A value outside the fp16 range became +-inf (or was NaN): record it, so
  // the caller learns of it instead of receiving silent infinities.  Rows past
  // M are zero-filled operands, hence finite, and are never stored anyway.
  if (p.out_f16 && __any_sync(0xffffffffu, nonfinite != 0u) && lane == 0 && p.err) atomicOr(p.err, kErrRange);
}

// SwiGLU drain of one accumulator: columns [0, 128) hold gate, [128, 256) the
// matching up.  Output columns col_base + j, j < 128, in two 64-column boxes;
// gate bias at bias[col], up bias at bias[up_off + col].
__device__ __forceinline__ void epilogue_swiglu(const GemmArgs& p, const CUtensorMap* omap, uint32_t taddr, int row0,
                                                int lane, int g, int col_base, uint8_t* stage, uint32_t& nbox) {
  const uint16_t* bias = p.bias ? p.bias + int64_t(g) * p.bias_gstride : nullptr;
  const int n_left = p.N - col_base;
  const int boxes = n_left >= 128 ? 2 : (n_left > 0 ? (n_left + 63) / 64 : 0);  // warp-uniform
  for (int b = 0; b < boxes; ++b) {
    uint8_t* buf = next_buf(stage, nbox, lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t rg[16], ru[16];
      __syncwarp();
      tmem_ld16x2_sync(taddr + uint32_t(b * 64 + q * 16), rg, taddr + uint32_t(128 + b * 64 + q * 16), ru);
      const int col0 = col_base + b * 64 + q * 16;
      float gv[16], uv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        gv[j] = __uint_as_float(rg[j]);
        uv[j] = __uint_as_float(ru[j]);
      }
      if (bias != nullptr) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (col0 + 8 * h < p.N) {
            const uint4 bg = __ldg(reinterpret_cast<const uint4*>(bias + col0) + h);
            const uint4 bu = __ldg(reinterpret_cast<const uint4*>(bias + p.up_off + col0) + h);
            const uint32_t wg[4] = {bg.x, bg.y, bg.z, bg.w};
            const uint32_t wu[4] = {bu.x, bu.y, bu.z, bu.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              gv[8 * h + 2 * j] += bf16_lo(wg[j]);
              gv[8 * h + 2 * j + 1] += bf16_hi(wg[j]);
              uv[8 * h + 2 * j] += bf16_lo(wu[j]);
              uv[8 * h + 2 * j + 1] += bf16_hi(wu[j]);
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 o;
        o.x = pack_bf16x2(silu(gv[8 * h + 0]) * uv[8 * h + 0], silu(gv[8 * h + 1]) * uv[8 * h + 1]);
        o.y = pack_bf16x2(silu(gv[8 * h + 2]) * uv[8 * h + 2], silu(gv[8 * h + 3]) * uv[8 * h + 3]);
        o.z = pack_bf16x2(silu(gv[8 * h + 4]) * uv[8 * h + 4], silu(gv[8 * h + 5]) * uv[8 * h + 5]);
        o.w = pack_bf16x2(silu(gv[8 * h + 6]) * uv[8 * h + 6], silu(gv[8 * h + 7]) * uv[8 * h + 7]);
        stage16(buf, lane, q * 2 + h, o);
      }
    }
    store_box(omap, buf, lane, col_base + b * 64, row0, g, p.M);
  }
}

// ============================================================================
// Single-CTA kernel
// ============================================================================
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap omap, const GemmArgs p) {
  using C = Cta1<BN>;
  constexpr int kStages1 = C::kStages;
  constexpr int kStageBytes1 = C::kStageBytes;
  // SwiGLU tiles take two 128-row weight boxes: only the 256-wide tile has room
  const bool swiglu = BN == 256 && p.swiglu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + kStages1;
  uint64_t* tfull = empty + kStages1;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int out_bn = swiglu ? BN / 2 : BN;  // output columns per tile
  const int m_tiles = (p.M + BM1 - 1) / BM1;
  const int n_tiles = (p.N + out_bn - 1) / out_bn;
  const int tiles = m_tiles * n_tiles * p.groups;
  const int k_iters = p.k_blocks * p.kshards;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages1; ++s) {
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
    tma_prefetch_desc(&omap);
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
          uint8_t* sa = smem + stage * kStageBytes1;
          mbar_arrive_expect_tx(&full[stage], kStageBytes1);
          if (p.a_split_input)
            tma_load_3d(sa, &amap, &full[stage], kb * BK, s, tc.mb * BM1);
          else
            tma_load_3d(sa, &amap, &full[stage], kb * BK, tc.mb * BM1, p.a_follows_shard ? s : 0);
          if (swiglu) {  // two 128-row boxes: gate rows, then the matching up rows
            tma_load_3d(sa + kABytes1, &bmap, &full[stage], kb * BK, tc.nb * 128, tc.g + s);
            tma_load_3d(sa + kABytes1 + 128 * BK * 2, &bmap, &full[stage], kb * BK, int(p.up_off) + tc.nb * 128,
                        tc.g + s);
          } else {
            tma_load_3d(sa + kABytes1, &bmap, &full[stage], kb * BK, tc.nb * BN, tc.g + s);
          }
          ++issued;
          if (++stage == kStages1) {
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
        for (int s = 0; s < kStages1; ++s) {
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
          const uint32_t sa = smem_u32(smem + stage * kStageBytes1);
          const uint64_t da = sdesc_sw128(sa, 16, 1024);
          const uint64_t db = sdesc_sw128(sa + kABytes1, 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // advance 16 bf16 = 32 bytes inside the swizzle row
            umma_ss(d_tmem, da + uint64_t(2 * k), db + uint64_t(2 * k), C::kIdesc, (it | k) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == kStages1) {
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
    uint8_t* stage = smem + C::kEpiOff + (warp - 2) * 2 * kEpiBuf;
    uint32_t nbox = 0;
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
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kAccCols);
      const int row0 = tc.mb * BM1 + q * 32;
      if (swiglu)
        epilogue_swiglu(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, stage, nbox);
      else if (p.out_f32)
        epilogue_rows_f32(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, out_bn, stage, nbox);
      else
        epilogue_rows(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, out_bn, stage, nbox);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if (!ok && lane == 0) report_timeout(p.err, abort_flag);
    if (lane == 0) bulk_wait_all();  // this warp's TMA stores are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ============================================================================
// CTA-pair kernel (cluster of 2, tcgen05 cta_group::2)
// ============================================================================
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                     const __grid_constant__ CUtensorMap omap, const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff2);  // the leader's copy is the one used
  uint64_t* empty = full + kStages2;                               // both CTAs' copies used
  uint64_t* tfull = empty + kStages2;                              // both
  uint64_t* tempty = tfull + 2;                                    // the leader's copy used
  uint64_t* drain = tempty + 2;
  uint64_t* exit_bar = drain + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(exit_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader, 1 = peer
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int out_bn = p.swiglu ? BN2 / 2 : BN2;  // output columns per tile
  const int m_tiles = (p.M + BM2 - 1) / BM2;
  const int n_tiles = (p.N + out_bn - 1) / out_bn;
  const int tiles = m_tiles * n_tiles * p.groups;
  const int k_iters = p.k_blocks * p.kshards;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&full[s], 1);   // the leader's producer arrives (+ both CTAs' TMA bytes)
      mbar_init(&empty[s], 1);  // one multicast commit per use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);   // one multicast commit per use
      mbar_init(&tempty[a], 8);  // four epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    mbar_init(exit_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
    tma_prefetch_desc(&omap);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int64_t issued = 0;
      for (int t = pair; t < tiles && ok; t += n_pairs) {
        const TileCoord tc = decode_tile(t, m_tiles, n_tiles);
        for (int it = 0; it < k_iters; ++it) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int s = it / p.k_blocks;
          const int kb = it - s * p.k_blocks;
          uint8_t* sa = smem + stage * kStageBytes2;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes2);  // both CTAs' bytes
          const int a_row = tc.mb * BM2 + int(rank) * 128;
          if (p.a_split_input)
            tma_load_3d_pair(sa, &amap, fb, kb * BK, s, a_row);
          else
            tma_load_3d_pair(sa, &amap, fb, kb * BK, a_row, p.a_follows_shard ? s : 0);
          // B: this CTA's 128 rows of the 256-row tile; SwiGLU: the even CTA
          // fetches the gate rows, the odd one the matching up rows.
          const int b_row = p.swiglu ? int(rank) * int(p.up_off) + tc.nb * 128 : tc.nb * BN2 + int(rank) * 128;
          tma_load_3d_pair(sa + kHalfBytes, &bmap, fb, kb * BK, b_row, tc.g + s);
          ++issued;
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) report_timeout(p.err, abort_flag);
      // Tail: every stage this CTA filled must be released (the MMAs reading it
      // done and the commit arrived here) before the CTA may exit.  Bounded.
      const volatile int no_abort = 0;
      for (int s = 0; s < kStages2; ++s) {
        if (issued <= s) break;
        // stage s was last filled in the current round if s < stage, else in the previous one
        mbar_wait(&empty[s], s < stage ? phase : (phase ^ 1u), ok ? abort_flag : &no_abort);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += n_pairs, ++local) {
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
          const uint32_t sa = smem_u32(smem + stage * kStageBytes2);
          const uint64_t da = sdesc_sw128(sa, 16, 1024);
          const uint64_t db = sdesc_sw128(sa + kHalfBytes, 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_ss_pair(d_tmem, da + uint64_t(2 * k), db + uint64_t(2 * k), kIdesc2, (it | k) != 0 ? 1u : 0u);
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(&tfull[acc], 0x3);
      }
      const volatile int no_abort = 0;
      if (!ok) {
        report_timeout(p.err, abort_flag);
        umma_commit_pair_mc(drain, 0x1);
        mbar_wait(drain, 0, &no_abort);
      } else {
        // Tail: both CTAs' epilogues have released the last accumulators (their
        // arrivals, some remote, have landed here) before the leader may exit.
        for (int i = local - 2 < 0 ? 0 : local - 2; i < local; ++i)
          mbar_wait(&tempty[i & 1], (i >> 1) & 1, abort_flag);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    uint8_t* stage = smem + kEpiOff2 + (warp - 2) * 2 * kEpiBuf;
    uint32_t nbox = 0;
    int local = 0;
    bool ok = true;
    for (int t = pair; t < tiles; t += n_pairs, ++local) {
      const TileCoord tc = decode_tile(t, m_tiles, n_tiles);
      const int acc = local & 1;
      if (!mbar_wait(&tfull[acc], (local >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kAccCols);
      const int row0 = tc.mb * BM2 + int(rank) * 128 + q * 32;
      if (p.swiglu)
        epilogue_swiglu(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, stage, nbox);
      else if (p.out_f32)
        epilogue_rows_f32(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, out_bn, stage, nbox);
      else
        epilogue_rows(p, &omap, taddr, row0, lane, tc.g, tc.nb * out_bn, out_bn, stage, nbox);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + uint32_t(acc * sizeof(uint64_t)));
    }
    if (!ok && lane == 0) report_timeout(p.err, abort_flag);
    if (lane == 0) bulk_wait_all();  // this warp's TMA stores are complete before the CTA exits
  }

  // Exit handshake: neither CTA leaves while the other may still signal its
  // barriers.  Bounded like every other wait.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(mapa_shared(smem_u32(exit_bar), rank ^ 1u));
    const volatile int no_abort = 0;
    if (!mbar_wait(exit_bar, 0, &no_abort)) report_timeout(p.err, abort_flag);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

int g_max_pairs[64] = {};
std::mutex g_pairs_mu;

// Pair clusters of the pair kernel that fit on device `dev` at once (cached).
int device_max_pairs(int dev) {
  std::lock_guard<std::mutex> lock(g_pairs_mu);
  if (g_max_pairs[dev] == 0) {
    int num_sms = 0;
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms < 2)
      num_sms = 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(num_sms & ~1));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes2;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg) != cudaSuccess || n <= 0) n = num_sms / 2;
    g_max_pairs[dev] = n;
  }
  return g_max_pairs[dev];
}

}  // namespace

int gemm_max_active_pairs(int num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
  const int pairs = device_max_pairs(dev);
  // a launch given part of the SMs (beside another kernel) stays within them
  return pairs < num_sms / 2 ? pairs : (num_sms / 2 > 0 ? num_sms / 2 : 1);
}

namespace {

// A's map: {K_s, rows, z}, or {K_s, z, rows} for a split input (memory
// [rows][z][K_s]), with a box of 64 x box_rows rows either way.
CUresult make_a_map(CUtensorMap* map, const GemmOperand& A, const GemmArgs& a, uint32_t box_rows) {
  if (a.a_split_input) return make_map_3d_bf16_box(map, A.base, A.k, A.z, A.rows, BK, 1, box_rows);
  return make_map_3d_bf16(map, A.base, A.k, A.rows, A.z, BK, box_rows, A.zrows);
}

// One-CTA kernel with 128 x BN tiles, one CTA per SM at most.
template <int BN>
cudaError_t launch_cta1(const GemmOperand& A, const GemmOperand& B, const GemmArgs& a, CUtensorMap& amap,
                        const CUtensorMap& omap, int num_sms, cudaStream_t s) {
  using C = Cta1<BN>;
  const bool swiglu = BN == 256 && a.swiglu;
  if (a.swiglu && !swiglu) return note_cuda_error("gemm: SwiGLU needs 256-column tiles", cudaErrorInvalidValue);
  const int out_bn = swiglu ? BN / 2 : BN;
  CUtensorMap bmap;
  if (make_a_map(&amap, A, a, BM1) != CUDA_SUCCESS ||
      make_map_3d_bf16(&bmap, B.base, B.k, B.rows, B.z, BK, uint32_t(out_bn), B.zrows) != CUDA_SUCCESS)
    return note_cuda_error("gemm: tensor map encode", cudaErrorInvalidValue);
  const int64_t tiles = int64_t((a.M + BM1 - 1) / BM1) * ((a.N + out_bn - 1) / out_bn) * a.groups;
  const int grid = int(tiles < num_sms ? tiles : num_sms);
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return note_cuda_error("gemm: set shared memory size", e);
  gemm_tc_kernel<BN><<<grid, kThreads, C::kSmemBytes, s>>>(amap, bmap, omap, a);
  count_launch();
  return note_cuda_error("gemm: launch", cudaGetLastError());
}

}  // namespace

cudaError_t launch_gemm(const GemmOperand& A, const GemmOperand& B, const GemmArgs& a, int num_sms,
                        cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.groups <= 0) return cudaSuccess;
  CUtensorMap amap, omap;
  const CUresult om = a.out_f32 ? make_map_out_f32(&omap, a.out, uint64_t(a.N), uint64_t(a.M), uint64_t(a.groups),
                                                   uint64_t(a.ldo), uint64_t(a.out_gstride))
                                : make_map_out_u16(&omap, a.out, uint64_t(a.N), uint64_t(a.M), uint64_t(a.groups),
                                                   uint64_t(a.ldo), uint64_t(a.out_gstride));
  if (om != CUDA_SUCCESS) return note_cuda_error("gemm: output tensor map encode", cudaErrorInvalidValue);
  const int plan = gemm_tile_plan(a.M, a.N, a.groups, a.swiglu != 0, num_sms);
  if (plan == kPlanPair) {
    // CTA-pair kernel: each CTA loads 128-row halves of both operands.
    CUtensorMap bmap;
    if (make_a_map(&amap, A, a, 128) != CUDA_SUCCESS ||
        make_map_3d_bf16(&bmap, B.base, B.k, B.rows, B.z, BK, 128, B.zrows) != CUDA_SUCCESS)
      return note_cuda_error("gemm (CTA pairs): tensor map encode", cudaErrorInvalidValue);
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes2);
    if (e != cudaSuccess) return note_cuda_error("gemm (CTA pairs): set shared memory size", e);
    const int out_bn = a.swiglu ? BN2 / 2 : BN2;
    const int64_t tiles = int64_t((a.M + BM2 - 1) / BM2) * ((a.N + out_bn - 1) / out_bn) * a.groups;
    int pairs = gemm_max_active_pairs(num_sms);
    if (tiles < pairs) pairs = int(tiles);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(2 * pairs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes2;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel, amap, bmap, omap, a);
    count_launch();
    if (e == cudaSuccess) e = cudaGetLastError();
    return note_cuda_error("gemm (CTA pairs): launch", e);
  }
  return plan == kPlanCta128x128 ? launch_cta1<128>(A, B, a, amap, omap, num_sms, s)
                                 : launch_cta1<256>(A, B, a, amap, omap, num_sms, s);
}

}  // namespace tp
