// attn.cu - a6, per-shard scaled dot-product attention on tcgen05.
//
// Under tensor parallelism the colwise Q/K/V projections give each rank a
// subset of the heads (Diffusers "Tensor parallelism" page, section "Colwise
// and rowwise", paragraph on attention), so attention runs independently per
// (shard, head).  For every head j of shard r:
//     O = softmax(Q K^T / sqrt(128)) V     (non-causal, no mask)
// computed with an online softmax over 128-key tiles.
//
// Structure: one CTA per (shard, head, 256 query rows) = two 128-row query
// tiles t = 0, 1, 576 threads:
//   warps 0-15 softmax, eight per tile.  TMEM lets warp w reach lanes
//              32*(w%4)..+31, so warps w and w+4 share the same 32 query rows:
//              each takes one half (64 columns) of those rows' scores.  The
//              two halves exchange their partial row maxima through shared
//              memory behind a per-tile mbarrier; every thread then applies
//              the same running max.  p = 2^(s*log2(e)/sqrt(d) - m) with the
//              hardware ex2, element-wise arithmetic on packed fp32 pairs; the
//              P of a half (fp16 pairs) is written over the first 32 columns of
//              that half's own S region; O is rescaled in TMEM only when the
//              running max grows by more than 8 (log2 units) - otherwise the
//              stale max is kept for both O and the row sum, which leaves O/l
//              unchanged.  Each half keeps its own partial row sum; the two are
//              added at the end, and each half normalises and stores its 64
//              output columns.
//   warp 16    TMA producer: Q0, Q1 once, then K and V tiles into two 2-stage
//              rings, K one tile ahead of V.
//   warp 17    TMEM allocator + MMA issuer, in the order
//                S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//              so that while one tile's softmax runs the tensor core works on
//              the other tile.  S = Q K^T reads both operands from shared
//              memory (K-major); O += P V reads P from TMEM (keys 0-63 from the
//              first S half, 64-127 from the second) and V from shared memory as
//              an MN-major operand.  tcgen05 MMAs of one thread execute in issue
//              order, so S_t(j+1) cannot overwrite P_t(j) before PV_t(j) has read
//              it, and when S_t(j) is signalled complete PV_t(j-1) has finished
//              updating O_t (safe to rescale).
// TMEM columns: S0 [0,128) with P0 in [0,32) + [64,96), S1 [128,256) likewise,
// O0 [256,384), O1 [384,512).
//
// Precision: Q, K, V arrive in fp16 and P is rounded to fp16 (11-bit
// significand; |Q|, |K|, |V| of a unit-variance projection stay far below the
// fp16 limit, and P <= 2^8 by the rescale rule), because bf16's 8-bit
// significand at these two points alone costs more than the stated max-error
// budget of the block.  S, the row statistics and O accumulate in fp32; O is
// written in bf16 for the out-projection.
// Every mbarrier wait is bounded (ptx.cuh); a timeout drains and exits.
#include <cuda_bf16.h>

#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

constexpr int kD = 128;             // head dim
constexpr int kBQ = 128;            // query rows per tile
constexpr int kTiles = 2;           // query tiles per CTA
constexpr int kBKV = 128;           // keys per KV tile
constexpr int kBox = 128 * 64 * 2;  // one TMA box: 128 rows x 64 fp16 (16 KB)
constexpr int kQBytes = 2 * kBox;   // one Q tile: d in two 64-column boxes
constexpr int kKBytes = 2 * kBox;   // one K tile (d in two boxes)
constexpr int kVBytes = 2 * kBox;   // one V tile
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kThreads = 576;
constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kQOff = 0;
constexpr int kKOff = kTiles * kQBytes;
constexpr int kVOff = kKOff + kKStages * kKBytes;
constexpr int kXchOff = kVOff + kVStages * kVBytes;  // row-max exchange [tile][slot][half][128] + row sums [tile][half][128]
constexpr int kXchBytes = (kTiles * 2 * 2 + kTiles * 2) * kBQ * 4;
constexpr int kBarOff = kXchOff + kXchBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kColS0 = 0, kColO0 = 256;  // tile t: S at kColS0 + 128 t, O at kColO0 + 128 t
constexpr uint32_t kIdescS = idesc_f32acc(kBQ, kBKV, false, false);  // fp16 Q, K
constexpr uint32_t kIdescPV = idesc_f32acc(kBQ, kD, false, true);    // fp16 P, V; B (= V) is MN-major
constexpr float kRescaleThreshold = 8.0f;                           // log2 units

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// 576 threads: eighteen warps, so some SM sub-partitions (16K registers each)
// hold five of them, which caps a thread at about 100 registers.
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qkv, const AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [3]
  uint64_t* k_empty = bars + 4;   // [3]
  uint64_t* v_full = bars + 7;    // [2]
  uint64_t* v_empty = bars + 9;   // [2]
  uint64_t* s_full = bars + 11;   // [2] per query tile
  uint64_t* p_full = bars + 13;   // [2] per query tile
  uint64_t* o_done = bars + 15;   // [2] per query tile (after the last P.V)
  uint64_t* drain = bars + 17;
  uint64_t* xch = bars + 18;      // [2] per query tile: both halves' partial maxima written
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 20);
  float* xmax = reinterpret_cast<float*>(smem + kXchOff);  // [tile][slot][half][row]
  float* xsum = xmax + kTiles * 2 * 2 * kBQ;                // [tile][half][row]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qb = blockIdx.x;
  const int shard = blockIdx.y / p.Hs;
  const int head = blockIdx.y - shard * p.Hs;
  const int n_kv = (p.M + kBKV - 1) / kBKV;
  const int qcol = head * kD;
  const int kcol = (p.Hs + head) * kD;
  const int vcol = (2 * p.Hs + head) * kD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 8);  // the eight softmax warps of that tile
      mbar_init(&o_done[s], 1);
      mbar_init(&xch[s], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&qkv);
      mbar_arrive_expect_tx(q_full, kTiles * kQBytes);
      for (int t = 0; t < kTiles; ++t) {
        uint8_t* sq = smem + kQOff + t * kQBytes;
        const int row = qb * (kTiles * kBQ) + t * kBQ;
        tma_load_3d(sq, &qkv, q_full, qcol, row, shard);
        tma_load_3d(sq + kBox, &qkv, q_full, qcol + 64, row, shard);
      }
      // Order K_0, then (K_{j+1}, V_j) for each j: the MMA order is
      // S(j) [K_j], PV(j) [V_j], S(j+1) [K_{j+1}], so K runs one tile ahead.
      bool ok = true;
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int j) -> bool {
        const int st = j % kKStages;
        if (!mbar_wait(&k_empty[st], ((j / kKStages) & 1) ^ 1u, abort_flag)) return false;
        uint8_t* sk = smem + kKOff + st * kKBytes;
        mbar_arrive_expect_tx(&k_full[st], kKBytes);
        tma_load_3d(sk, &qkv, &k_full[st], kcol, j * kBKV, shard);
        tma_load_3d(sk + kBox, &qkv, &k_full[st], kcol + 64, j * kBKV, shard);
        ++k_issued;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&v_empty[st], ((j >> 1) & 1) ^ 1u, abort_flag)) return false;
        uint8_t* sv = smem + kVOff + st * kVBytes;
        mbar_arrive_expect_tx(&v_full[st], kVBytes);
        tma_load_3d(sv, &qkv, &v_full[st], vcol, j * kBKV, shard);
        tma_load_3d(sv + kBox, &qkv, &v_full[st], vcol + 64, j * kBKV, shard);
        ++v_issued;
        return true;
      };
      ok = load_k(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv && !load_k(j + 1)) ok = false;
        if (ok && !load_v(j)) ok = false;
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        const volatile int no_abort = 0;
        mbar_wait(q_full, 0, &no_abort);
        // the last loads issued may still be landing
        for (int j = k_issued - kKStages < 0 ? 0 : k_issued - kKStages; j < k_issued; ++j)
          mbar_wait(&k_full[j % kKStages], (j / kKStages) & 1, &no_abort);
        for (int j = v_issued - 2 < 0 ? 0 : v_issued - 2; j < v_issued; ++j)
          mbar_wait(&v_full[j & 1], (j >> 1) & 1, &no_abort);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sq0 = smem_u32(smem + kQOff);
      auto issue_s = [&](int t, int j) {
        const uint32_t sq = sq0 + uint32_t(t * kQBytes);
        const uint32_t sk = smem_u32(smem + kKOff + (j % kKStages) * kKBytes);
        const uint32_t d = tmem_base + kColS0 + uint32_t(t * 128);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = uint32_t((kk >> 2) * kBox + (kk & 3) * 32);
          umma_ss(d, sdesc_sw128(sq + off, 16, 1024), sdesc_sw128(sk + off, 16, 1024), kIdescS, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t sv = smem_u32(smem + kVOff + (j & 1) * kVBytes);
        const uint32_t d = tmem_base + kColO0 + uint32_t(t * 128);
        const uint32_t a = tmem_base + kColS0 + uint32_t(t * 128);
#pragma unroll
        for (int kk = 0; kk < kBKV / 16; ++kk) {
          // 16 keys per step: P of keys 0-63 in columns [0,32), of keys 64-127 in
          // [64,96) (fp16 pairs); rows kk*16.. of both V boxes
          const uint32_t pcol = uint32_t((kk >> 2) * 64 + (kk & 3) * 8);
          umma_ts(d, a + pcol, sdesc_sw128(sv + uint32_t(kk * 16 * 128), kBox, 1024), kIdescPV,
                  (j | kk) != 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&k_empty[0]);  // K_0 no longer read once these complete
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const bool more = j + 1 < n_kv;
        // tile 0
        if (!mbar_wait(&p_full[0], j & 1, abort_flag) || !mbar_wait(&v_full[j & 1], (j >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(0, j);
        if (!more) umma_commit(&o_done[0]);
        if (more) {
          if (!mbar_wait(&k_full[(j + 1) % kKStages], ((j + 1) / kKStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(0, j + 1);
        }
        // tile 1
        if (!mbar_wait(&p_full[1], j & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(1, j);
        if (!more) umma_commit(&o_done[1]);
        umma_commit(&v_empty[j & 1]);  // V_j no longer read once these complete
        if (more) {
          issue_s(1, j + 1);
          umma_commit(&k_empty[(j + 1) % kKStages]);  // K_{j+1} done
        }
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        const volatile int no_abort = 0;
        umma_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-15)
    const int t = warp >> 3;                                     // query tile
    const int h = (warp >> 2) & 1;                               // column half of the scores
    const int rl = (warp & 3) * 32 + lane;                       // row within the tile (= TMEM lane)
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;  // TMEM lane quarter
    const uint32_t colS = kColS0 + uint32_t(t * 128 + 64 * h);   // this half's S (and P) columns
    const uint32_t colO = kColO0 + uint32_t(t * 128 + 64 * h);   // this half's O columns
    const int row = qb * (kTiles * kBQ) + t * kBQ + rl;
    float m_run = -INFINITY;  // running max (log2-scaled units) used for O and l
    float l_run = 0.f;        // this half's partial row sum
    bool ok = true;
    const float sl2 = p.scale_log2;
    const uint32_t ta = tmem_base + lane_off + colS;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kv0 = j * kBKV + 64 * h;
      const bool ragged = kv0 + 64 > p.M;  // keys >= M do not exist
      // Pass 1: this half's row max (two loads in flight, eight max chains).
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(ta, r0);
        tmem_ld32(ta + 32, r1);
        tmem_ld_wait();
        reg_fence32(r0);
        reg_fence32(r1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float v0 = __uint_as_float(r0[i]), v1 = __uint_as_float(r1[i]);
          if (ragged) {
            if (kv0 + i >= p.M) v0 = -INFINITY;
            if (kv0 + 32 + i >= p.M) v1 = -INFINITY;
          }
          mx8[i & 7] = fmaxf(mx8[i & 7], fmaxf(v0, v1));
        }
      }
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // Exchange the partial maxima of the two halves (slot j&1: a half can run
      // at most one step ahead of its partner, so the slot it writes is free).
      float* slot = xmax + ((t * 2 + (j & 1)) * 2) * kBQ;
      slot[h * kBQ + rl] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xch[t]);
      if (!mbar_wait(&xch[t], j & 1, abort_flag)) {
        ok = false;
        break;
      }
      mx = fmaxf(mx, slot[(h ^ 1) * kBQ + rl]) * sl2;
      if (j == 0) {
        m_run = mx;
      } else {
        // Both halves see the same maxima, so they take the same decision.  Rescale
        // only rows whose max grew by more than the threshold; the TMEM accesses are
        // warp-collective, so the whole warp takes the branch if any lane needs it
        // (other lanes scale by 1).  O_t already holds P_t(j-1) V.
        const bool need = mx > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_run - mx) : 1.0f;
          if (need) {
            m_run = mx;
            l_run *= alpha;
          }
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[16];
            const uint32_t to = tmem_base + lane_off + colO + uint32_t(c * 16);
            tmem_ld16_sync(to, r);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(to, r);
          }
        }
      }
      // Pass 2: p = 2^(s*scale - m), 32 scores at a time on packed fp32 pairs.
      // P chunk c goes to columns [16c, 16c+16) of this half's region, which only
      // hold scores this thread has already read.
      const uint64_t scale2 = f32x2(sl2, sl2);
      const uint64_t negm2 = f32x2(-m_run, -m_run);
      uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32_sync(ta + uint32_t(c * 32), r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f32x2_split(fma_f32x2(f32x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), scale2, negm2),
                      x0, x1);
          if (ragged) {
            if (kv0 + c * 32 + 2 * i >= p.M) x0 = -INFINITY;
            if (kv0 + c * 32 + 2 * i + 1 >= p.M) x1 = -INFINITY;
          }
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          ls2[i & 3] = add_f32x2(ls2[i & 3], f32x2(p0, p1));
          pk[i] = pack_f16x2(p0, p1);
        }
        tmem_st16(ta + uint32_t(c * 16), pk);
      }
      {
        float a0, a1, b0, b1, c0, c1, d0, d1;
        f32x2_split(ls2[0], a0, a1);
        f32x2_split(ls2[1], b0, b1);
        f32x2_split(ls2[2], c0, c1);
        f32x2_split(ls2[3], d0, d1);
        l_run += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok) ok = mbar_wait(&o_done[t], 0, abort_flag);
    if (ok) {
      // total row sum = both halves' partial sums (one more exchange phase)
      float* xs = xsum + t * 2 * kBQ;
      xs[h * kBQ + rl] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xch[t]);
      ok = mbar_wait(&xch[t], n_kv & 1, abort_flag);
      if (ok) l_run += xs[(h ^ 1) * kBQ + rl];
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      uint16_t* orow = p.out + (int64_t(shard) * p.M + row) * int64_t(p.Hs * kD) + head * kD + 64 * h;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32_sync(tmem_base + lane_off + colO + uint32_t(c * 32), r);
        uint4 o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[i].x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l);
          o[i].y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l);
          o[i].z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l);
          o[i].w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l);
        }
        if (row < p.M) {
          uint4* op = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) op[i] = o[i];
        }
      }
    }
    if (!ok && lane == 0) report_timeout(p.err, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    y[i] = exp2_poly(x[i]);
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  exp2_poly_kernel<<<unsigned(blocks), 256, 0, s>>>(x, y, n);
  count_launch();
  return note_cuda_error("exp2_poly: launch", cudaGetLastError());
}

cudaError_t launch_attention(const CUtensorMap& qkv_map, const AttnArgs& a, cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  const int q_blocks = (a.M + kTiles * kBQ - 1) / (kTiles * kBQ);
  dim3 grid(static_cast<unsigned>(q_blocks), static_cast<unsigned>(a.T * a.Hs));
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return note_cuda_error("attention: set shared memory size", e);
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(qkv_map, a);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    cudaFuncAttributes fa{};
    char detail[160];
    if (cudaFuncGetAttributes(&fa, attn_tc_kernel) == cudaSuccess)
      snprintf(detail, sizeof(detail), "kernel: %d registers/thread, max %d threads/block, %zu B static smem",
               fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes);
    else
      snprintf(detail, sizeof(detail), "kernel attributes unavailable");
    return note_cuda_error("attention: launch", e, detail);
  }
  return cudaSuccess;
}

}  // namespace tp
