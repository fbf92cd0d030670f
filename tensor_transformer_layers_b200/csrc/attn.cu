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
// tiles t = 0, 1, 320 threads:
//   warps 0-3  softmax of tile 0, warps 4-7 softmax of tile 1: thread i of a
//              warpgroup owns query row i (its TMEM lane), so the row max and
//              row sum are per-thread reductions over the 128 scores it loads;
//              p = 2^(s*log2(e)/sqrt(d) - m) with the hardware ex2; P is packed
//              to fp16 pairs and written back over the first 64 columns of its
//              own S buffer; O is rescaled in TMEM only when the running max
//              grows by more than 8 (log2 units) - otherwise the stale max is
//              kept for both O and the row sum, which leaves O/l unchanged.
//   warp 8     TMA producer: Q0, Q1 once, then K and V tiles into a 2-stage ring.
//   warp 9     TMEM allocator + MMA issuer, in the order
//                S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//              so that while one warpgroup computes its softmax the tensor core
//              works on the other tile.  S = Q K^T reads both operands from
//              shared memory (K-major); O += P V reads P from TMEM and V from
//              shared memory as an MN-major operand.  tcgen05 MMAs of one
//              thread execute in issue order, so S_t(j+1) cannot overwrite P_t(j)
//              before PV_t(j) has read it, and when S_t(j) is signalled complete
//              PV_t(j-1) has finished updating O_t (safe to rescale).
// TMEM columns: S0/P0 [0,128), S1/P1 [128,256), O0 [256,384), O1 [384,512).
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
constexpr int kKVBytes = 4 * kBox;  // K tile (2 boxes) + V tile (2 boxes)
constexpr int kStages = 2;
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kQOff = 0;
constexpr int kKVOff = kTiles * kQBytes;
constexpr int kBarOff = kKVOff + kStages * kKVBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kColS0 = 0, kColO0 = 256;  // tile t: S at kColS0 + 128 t, O at kColO0 + 128 t
constexpr uint32_t kIdescS = idesc_f32acc(kBQ, kBKV, false, false);  // fp16 Q, K
constexpr uint32_t kIdescPV = idesc_f32acc(kBQ, kD, false, true);    // fp16 P, V; B (= V) is MN-major
constexpr float kRescaleThreshold = 8.0f;                           // log2 units

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// 320 threads: ten warps, so some SM sub-partitions (16K registers each) hold
// three of them, which caps a thread at 168 registers.
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qkv, const AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2] per query tile
  uint64_t* p_full = bars + 7;    // [2] per query tile
  uint64_t* o_done = bars + 9;    // [2] per query tile (after the last P.V)
  uint64_t* drain = bars + 11;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 12);
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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);  // the four warps of that tile's softmax warpgroup
      mbar_init(&o_done[s], 1);
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
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sk = smem + kKVOff + st * kKVBytes;
        mbar_arrive_expect_tx(&kv_full[st], kKVBytes);
        tma_load_3d(sk, &qkv, &kv_full[st], kcol, j * kBKV, shard);
        tma_load_3d(sk + kBox, &qkv, &kv_full[st], kcol + 64, j * kBKV, shard);
        tma_load_3d(sk + 2 * kBox, &qkv, &kv_full[st], vcol, j * kBKV, shard);
        tma_load_3d(sk + 3 * kBox, &qkv, &kv_full[st], vcol + 64, j * kBKV, shard);
        ++issued;
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        const volatile int no_abort = 0;
        mbar_wait(q_full, 0, &no_abort);
        // the last (up to) two tiles issued may still be landing
        for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
          mbar_wait(&kv_full[j & 1], (j >> 1) & 1, &no_abort);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors are computed once: a descriptor's low field is the start
      // address >> 4, so moving inside shared memory is an integer add.
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + kQOff), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(smem + kKVOff), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(smem + kKVOff + 2 * kBox), kBox, 1024);
      auto issue_s = [&](int t, int j) {
        const uint64_t dq = dq0 + uint64_t((t * kQBytes) >> 4);
        const uint64_t dk = dk0 + uint64_t(((j & 1) * kKVBytes) >> 4);
        const uint32_t d = tmem_base + kColS0 + uint32_t(t * 128);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = uint64_t(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
          umma_ss(d, dq + off, dk + off, kIdescS, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint64_t dv = dv0 + uint64_t(((j & 1) * kKVBytes) >> 4);
        const uint32_t d = tmem_base + kColO0 + uint32_t(t * 128);
        const uint32_t a = tmem_base + kColS0 + uint32_t(t * 128);
#pragma unroll
        for (int kk = 0; kk < kBKV / 16; ++kk) {
          // 16 keys per step: P columns kk*8.. (fp16 pairs); rows kk*16.. of both V boxes
          umma_ts(d, a + uint32_t(kk * 8), dv + uint64_t((kk * 16 * 128) >> 4), kIdescPV, (j | kk) != 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&kv_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const bool more = j + 1 < n_kv;
        // tile 0
        if (!mbar_wait(&p_full[0], j & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(0, j);
        if (!more) umma_commit(&o_done[0]);
        if (more) {
          if (!mbar_wait(&kv_full[st ^ 1], ((j + 1) >> 1) & 1, abort_flag)) {
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
        umma_commit(&kv_empty[st]);  // K_j and V_j no longer read once these complete
        if (more) issue_s(1, j + 1);
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        const volatile int no_abort = 0;
        umma_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int t = warp >> 2;                                     // query tile of this warpgroup
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;  // TMEM lane quarter
    const uint32_t colS = kColS0 + uint32_t(t * 128);
    const uint32_t colO = kColO0 + uint32_t(t * 128);
    const int row = qb * (kTiles * kBQ) + t * kBQ + (warp & 3) * 32 + lane;
    float m_run = -INFINITY;  // running max (log2-scaled units) used for O and l
    float l_run = 0.f;
    bool ok = true;
    const float sl2 = p.scale_log2;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBKV];
#pragma unroll
      for (int c = 0; c < kBKV / 32; ++c) {
        uint32_t r[32];
        tmem_ld32_sync(tmem_base + lane_off + colS + uint32_t(c * 32), r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * kBKV;
      if (kv0 + kBKV > p.M) {  // ragged last key tile: keys >= M do not exist
#pragma unroll
        for (int i = 0; i < kBKV; ++i)
          if (kv0 + i >= p.M) s[i] = -INFINITY;
      }
      // row max over 8 independent chains, combined at the end (a shorter
      // dependency chain than one running max over 128 values)
      float m8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) m8[a] = s[a];
#pragma unroll
      for (int i = 8; i < kBKV; ++i) m8[i & 7] = fmaxf(m8[i & 7], s[i]);
      float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mx *= sl2;
      if (j == 0) {
        m_run = mx;
      } else {
        // Rescale only rows whose max grew by more than the threshold; the TMEM
        // accesses are warp-collective, so the whole warp takes the branch if any
        // lane needs it (other lanes scale by 1).  O_t already holds P_t(j-1) V.
        const bool need = mx > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_run - mx) : 1.0f;
          if (need) {
            m_run = mx;
            l_run *= alpha;
          }
#pragma unroll 1
          for (int c = 0; c < kD / 16; ++c) {
            uint32_t r[16];
            const uint32_t ta = tmem_base + lane_off + colO + uint32_t(c * 16);
            tmem_ld16_sync(ta, r);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(ta, r);
          }
        }
      }
      float l4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums
#pragma unroll
      for (int c = 0; c < kBKV / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(s[c * 32 + 2 * i], sl2, -m_run));
          const float p1 = ex2_approx(fmaf(s[c * 32 + 2 * i + 1], sl2, -m_run));
          l4[i & 3] += p0 + p1;
          pk[i] = pack_f16x2(p0, p1);
        }
        tmem_st16(tmem_base + lane_off + colS + uint32_t(c * 16), pk);  // P over S's first 64 columns
      }
      l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok) ok = mbar_wait(&o_done[t], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      uint16_t* orow = p.out + (int64_t(shard) * p.M + row) * int64_t(p.Hs * kD) + head * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
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

}  // namespace

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
