// attn.cu - a6, per-shard scaled dot-product attention on tcgen05.
//
// Under tensor parallelism the colwise Q/K/V projections give each rank a
// subset of the heads (Diffusers "Tensor parallelism" page, section "Colwise
// and rowwise", paragraph on attention), so attention runs independently per
// (shard, head).  For every head j of shard r:
//     O = softmax(Q K^T / sqrt(128)) V     (non-causal, no mask)
// computed with an online softmax over 128-key tiles.  The same kernel serves
// the per-block step of Ring attention ("Context parallelism" page, section
// on Ring attention): queries and keys/values may come from different token
// sets (two tensor maps), and in the statistics mode the kernel writes O
// normalised over the block's keys, in fp16, with each row's log-sum-exp in
// fp32, which the merge over key blocks needs (merge.cu).
//
// Structure: a work item is (shard, head, 256 query rows) = two 128-row query
// tiles t = 0, 1.  The kernel is persistent: one CTA per SM walks the items
// blockIdx.x, blockIdx.x + gridDim.x, ..., so one item's last blocks and its
// output overlap the next item's Q/K/V loads and first S (launching a CTA per
// item left ~10 us of every 84 us CTA slot outside the key loop: start-up,
// the last block's chain and output, and the gap before the next CTA).
// 320 threads:
//   warps 0-3  softmax of tile 0, warps 4-7 softmax of tile 1: thread i of a
//              warpgroup owns query row i (its TMEM lane), so the row max and
//              row sum are per-thread reductions over the 128 scores it loads;
//              p = 2^(s*log2(e)/sqrt(d) - m) with the hardware ex2; P is packed
//              to fp16 pairs and written back over the first 64 columns of its
//              own S buffer; O is rescaled in TMEM only when the running max
//              grows by more than 8 (log2 units) - otherwise the stale max is
//              kept for both O and the row sum, which leaves O/l unchanged.
//              After an item's last block the warpgroup writes O_t / l.
//   warp 8     TMA producer: per item K/V block 0, then Q0 and Q1 (each once the
//              previous item's last S_t is done), then the other K/V blocks,
//              all K/V through one 2-stage ring.
//   warp 9     TMEM allocator + MMA issuer, in the order
//                S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//              so that while one warpgroup computes its softmax the tensor core
//              works on the other tile (at an item's last block: PV0 PV1, then
//              the next item's S0 S1).  S = Q K^T reads both operands from
//              shared memory (K-major); O += P V reads P from TMEM and V from
//              shared memory as an MN-major operand.  tcgen05 MMAs of one
//              thread execute in issue order, so S_t(j+1) cannot overwrite P_t(j)
//              before PV_t(j) has read it, and when S_t(j) is signalled complete
//              PV_t(j-1) has finished updating O_t (safe to rescale).  The next
//              item's first P.V (which overwrites O_t) waits for the softmax
//              warpgroup's first P of that item, which it stores only after it
//              has read out O_t of the previous item.
// TMEM columns: S0/P0 [0,128), S1/P1 [128,256), O0 [256,384), O1 [384,512).
//
// Precision: Q, K, V arrive in fp16 and P is rounded to fp16 (11-bit
// significand; |Q|, |K|, |V| of a unit-variance projection stay far below the
// fp16 limit, and P <= 2^8 by the rescale rule), because bf16's 8-bit
// significand at these two points alone costs more than the stated max-error
// budget of the block.  S, the row statistics and O accumulate in fp32; O is
// written in bf16 for the out-projection.  A Ring block's O is written in
// fp16: each row is a convex combination of fp16 rows of V, so it stays in
// fp16's range, and its rounding (at most 2^-11 relative) is an eighth of
// the bf16 rounding (2^-8) the merged output takes once.
// Every mbarrier wait is bounded (ptx.cuh); a timeout drains and exits.
#include <cuda_bf16.h>

#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

// Waits until no TMA store of this thread still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

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
constexpr int kOutBuf = 32 * 128;                  // one softmax warp's staging box: 32 rows x 64 bf16
constexpr int kOutOff = kKVOff + kStages * kKVBytes;  // 8 staging boxes, one per softmax warp
constexpr int kBarOff = kOutOff + 8 * kOutBuf;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kColS0 = 0, kColO0 = 256;  // tile t: S at kColS0 + 128 t, O at kColO0 + 128 t
constexpr uint32_t kIdescS = idesc_f32acc(kBQ, kBKV, false, false);  // fp16 Q, K
constexpr uint32_t kIdescPV = idesc_f32acc(kBQ, kD, false, true);    // fp16 P, V; B (= V) is MN-major
constexpr float kRescaleThreshold = 8.0f;                           // log2 units

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// The output staging boxes use the 128-byte swizzle (chunk ^ (row & 7)), which
// is defined relative to 1024-byte-aligned boxes.
static_assert(kOutOff % 1024 == 0 && kOutBuf % 1024 == 0, "output staging boxes must be 1024-byte aligned");

// Work item i (query block qb = i % q_blocks of head-slot hs = i / q_blocks,
// hs = shard * Hs + head); consecutive items share a head's K and V in L2.
struct AttnItem {
  int qb, shard, head;
};
__device__ __forceinline__ AttnItem attn_item(int i, int q_blocks, int Hs) {
  AttnItem it;
  const int hs = i / q_blocks;
  it.qb = i - hs * q_blocks;
  it.shard = hs / Hs;
  it.head = hs - it.shard * Hs;
  return it;
}

// 320 threads: ten warps, so some SM sub-partitions (16K registers each) hold
// three of them, which caps a thread at 168 registers.
// kStats: the statistics mode (fp16 O and log-sum-exp) is a separate
// instantiation, so the ordinary kernel carries none of its code.
template <bool kStats>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                   const __grid_constant__ CUtensorMap omap, const AttnArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars + 0;    // [2] per query tile: Q_t of the current item landed
  uint64_t* q_empty = bars + 2;   // [2] per query tile: the item's last S_t done, Q_t may be replaced
  uint64_t* kv_full = bars + 4;   // [2] per ring stage
  uint64_t* kv_empty = bars + 6;  // [2] per ring stage
  uint64_t* s_full = bars + 8;    // [2] per query tile
  uint64_t* p_full = bars + 10;   // [2] per query tile
  uint64_t* o_done = bars + 12;   // [2] per query tile (after an item's last P.V)
  uint64_t* drain = bars + 14;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Ordinary attention reads Q, K and V from one buffer (the Q, K, V heads of
  // a row side by side): one map and offsets fixed by Hs.  Only the Ring
  // block (statistics mode) takes keys and values from another token set.
  const CUtensorMap* kvm = kStats ? &kvmap : &qmap;
  const int Mk = kStats ? p.Mk : p.Mq;
  const int n_kv = (Mk + kBKV - 1) / kBKV;
  const int q_blocks = (p.Mq + kTiles * kBQ - 1) / (kTiles * kBQ);
  const int n_items = q_blocks * p.T * p.Hs;
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_items = blockIdx.x < n_items ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
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
      tma_prefetch_desc(&qmap);
      if (kStats) tma_prefetch_desc(&kvmap);
      bool ok = true;
      int g = 0;           // K/V blocks issued (ring position)
      int qn[2] = {0, 0};  // Q tiles issued per tile slot
      for (int k = 0; k < my_items && ok; ++k) {
        const AttnItem it = attn_item(int(blockIdx.x) + k * int(gridDim.x), q_blocks, p.Hs);
        const int qcol = (kStats ? p.q_col0 : 0) + it.head * kD;
        const int kcol = (kStats ? p.k_col0 : p.Hs * kD) + it.head * kD;
        const int vcol = (kStats ? p.v_col0 : 2 * p.Hs * kD) + it.head * kD;
        // K/V block 0 first (its ring stage frees early), then Q_0 and Q_1 (each
        // free once the previous item's last S_t is done), then the other blocks.
        for (int j = 0; j < n_kv && ok; ++j, ++g) {
          const int st = g & 1;
          if (!mbar_wait(&kv_empty[st], ((g >> 1) & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sk = smem + kKVOff + st * kKVBytes;
          mbar_arrive_expect_tx(&kv_full[st], kKVBytes);
          tma_load_3d(sk, kvm, &kv_full[st], kcol, j * kBKV, it.shard);
          tma_load_3d(sk + kBox, kvm, &kv_full[st], kcol + 64, j * kBKV, it.shard);
          tma_load_3d(sk + 2 * kBox, kvm, &kv_full[st], vcol, j * kBKV, it.shard);
          tma_load_3d(sk + 3 * kBox, kvm, &kv_full[st], vcol + 64, j * kBKV, it.shard);
          if (j == 0) {
            for (int t = 0; t < kTiles; ++t) {
              if (!mbar_wait(&q_empty[t], (k & 1) ^ 1u, abort_flag)) {
                ok = false;
                break;
              }
              uint8_t* sq = smem + kQOff + t * kQBytes;
              const int row = it.qb * (kTiles * kBQ) + t * kBQ;
              mbar_arrive_expect_tx(&q_full[t], kQBytes);
              tma_load_3d(sq, &qmap, &q_full[t], qcol, row, it.shard);
              tma_load_3d(sq + kBox, &qmap, &q_full[t], qcol + 64, row, it.shard);
              ++qn[t];
            }
          }
        }
      }
      if (!ok) {
        report_timeout(p.err, abort_flag);
        // copies still landing: the last Q of each tile slot, the last two K/V blocks
        const volatile int no_abort = 0;
        for (int t = 0; t < kTiles; ++t)
          if (qn[t] > 0) mbar_wait(&q_full[t], (qn[t] - 1) & 1, &no_abort);
        for (int b = g - 2 < 0 ? 0 : g - 2; b < g; ++b) mbar_wait(&kv_full[b & 1], (b >> 1) & 1, &no_abort);
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
      // S_t of global block b (item b / n_kv, key block b % n_kv); after an
      // item's last S_t, Q_t may be replaced by the next item's.
      auto issue_s = [&](int t, int b) {
        const uint64_t dq = dq0 + uint64_t((t * kQBytes) >> 4);
        const uint64_t dk = dk0 + uint64_t(((b & 1) * kKVBytes) >> 4);
        const uint32_t d = tmem_base + kColS0 + uint32_t(t * 128);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = uint64_t(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
          umma_ss(d, dq + off, dk + off, kIdescS, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
        if (b % n_kv == n_kv - 1) umma_commit(&q_empty[t]);
      };
      // O_t (+)= P_t V of global block b; the first block of an item overwrites O_t.
      auto issue_pv = [&](int t, int b) {
        const uint64_t dv = dv0 + uint64_t(((b & 1) * kKVBytes) >> 4);
        const uint32_t d = tmem_base + kColO0 + uint32_t(t * 128);
        const uint32_t a = tmem_base + kColS0 + uint32_t(t * 128);
        const int j = b % n_kv;
#pragma unroll
        for (int kk = 0; kk < kBKV / 16; ++kk) {
          // 16 keys per step: P columns kk*8.. (fp16 pairs); rows kk*16.. of both V boxes
          umma_ts(d, a + uint32_t(kk * 8), dv + uint64_t((kk * 16 * 128) >> 4), kIdescPV, (j | kk) != 0 ? 1u : 0u);
        }
        if (j == n_kv - 1) umma_commit(&o_done[t]);
      };
      // S_t of block b needs K/V of b (waited by the caller) and, on an item's
      // first block, the item's Q_t.
      auto wait_q = [&](int t, int b) {
        return b % n_kv != 0 || mbar_wait(&q_full[t], (b / n_kv) & 1, abort_flag);
      };
      const int total = my_items * n_kv;
      bool ok = true;
      if (total > 0) {
        ok = mbar_wait(&kv_full[0], 0, abort_flag) && wait_q(0, 0);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          ok = wait_q(1, 0);
        }
        if (ok) {
          tc_fence_after();
          issue_s(1, 0);
        }
      }
      for (int b = 0; b < total && ok; ++b) {
        const int st = b & 1;
        const bool more = b + 1 < total;
        if (more && (b + 1) % n_kv != 0) {
          // inside an item: PV0(b) S0(b+1) PV1(b) S1(b+1), so one tile's softmax
          // overlaps the other tile's MMAs
          if (!mbar_wait(&p_full[0], b & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(0, b);
          if (!mbar_wait(&kv_full[st ^ 1], ((b + 1) >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(0, b + 1);
          if (!mbar_wait(&p_full[1], b & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(1, b);
          umma_commit(&kv_empty[st]);  // K and V of block b no longer read once these complete
          issue_s(1, b + 1);
        } else {
          // an item's last block: both P.V first, then (if there is a next item)
          // its first S, which waits for that item's Q
          if (!mbar_wait(&p_full[0], b & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(0, b);
          if (!mbar_wait(&p_full[1], b & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(1, b);
          umma_commit(&kv_empty[st]);
          if (more) {
            if (!mbar_wait(&kv_full[st ^ 1], ((b + 1) >> 1) & 1, abort_flag) || !wait_q(0, b + 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(0, b + 1);
            if (!wait_q(1, b + 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(1, b + 1);
          }
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
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int t = warp >> 2;                                     // query tile of this warpgroup
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;  // TMEM lane quarter
    const uint32_t colS = kColS0 + uint32_t(t * 128);
    const uint32_t colO = kColO0 + uint32_t(t * 128);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int b = 0;  // global block index (phase of s_full / p_full)
    for (int k = 0; k < my_items && ok; ++k) {
      float m_run = -INFINITY;  // running max (log2-scaled units) used for O and l
      float l_run = 0.f;
      for (int j = 0; j < n_kv; ++j, ++b) {
        if (!mbar_wait(&s_full[t], b & 1, abort_flag)) {
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
        if (kv0 + kBKV > Mk) {  // ragged last key tile: keys >= Mk do not exist
#pragma unroll
          for (int i = 0; i < kBKV; ++i)
            if (kv0 + i >= Mk) s[i] = -INFINITY;
        }
        // Row max: 3-input max over four independent chains (64 instructions
        // for 128 scores, a short dependency chain).  The element-wise code
        // below uses packed fp32 pairs: measured on B200, scalar fp32
        // add/mul/fma/max issued at this rate by warps on all four SM
        // sub-partitions slow concurrent tcgen05 MMAs by a third or more (a
        // 128x128x16 MMA from 64 to ~95-106 cycles), while the packed forms,
        // MUFU, conversions and integer ALU work at the same rate do not.
        float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int q = 0; q < (kBKV - 4) / 2; ++q) m4[q & 3] = fmax3(m4[q & 3], s[4 + 2 * q], s[5 + 2 * q]);
        float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
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
            const uint64_t alpha2 = f32x2(alpha, alpha);
#pragma unroll 1
            for (int c = 0; c < kD / 16; ++c) {
              uint32_t r[16];
              const uint32_t ta = tmem_base + lane_off + colO + uint32_t(c * 16);
              tmem_ld16_sync(ta, r);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float lo, hi;
                f32x2_split(mul_f32x2(f32x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), alpha2), lo, hi);
                r[2 * i] = __float_as_uint(lo);
                r[2 * i + 1] = __float_as_uint(hi);
              }
              tmem_st16(ta, r);
            }
          }
        }
        // p = 2^(s * sl2 - m) on pairs; row sum in two packed partial sums
        const uint64_t sl2x2 = f32x2(sl2, sl2), negm2 = f32x2(-m_run, -m_run);
        uint64_t l2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < kBKV / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f32x2_split(fma_f32x2(f32x2(s[c * 32 + 2 * i], s[c * 32 + 2 * i + 1]), sl2x2, negm2), x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            l2[i & 1] = add_f32x2(l2[i & 1], f32x2(p0, p1));
            pk[i] = pack_f16x2(p0, p1);
          }
          tmem_st16(tmem_base + lane_off + colS + uint32_t(c * 16), pk);  // P over S's first 64 columns
        }
        float la, lb;
        f32x2_split(add_f32x2(l2[0], l2[1]), la, lb);
        l_run += la + lb;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
      }
      // Epilogue of this item: O_t / l.  It reads O_t before this warp's next
      // p_full arrival, and the next item's first P.V (which overwrites O_t)
      // waits for that arrival.
      if (ok) ok = mbar_wait(&o_done[t], k & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        const AttnItem it = attn_item(int(blockIdx.x) + k * int(gridDim.x), q_blocks, p.Hs);
        const int row0 = it.qb * (kTiles * kBQ) + t * kBQ + (warp & 3) * 32;
        const float inv_l = 1.0f / l_run;
        const uint64_t inv_l2 = f32x2(inv_l, inv_l);
        uint8_t* stg = smem + kOutOff + warp * kOutBuf;
        // O_t / l, 64 columns at a time (bf16; fp16 in the statistics mode),
        // staged in this warp's box in the 128-byte swizzle of the output
        // map, then one TMA store (whole 128-byte lines; rows >= Mq are
        // clipped, a box wholly below Mq skipped).
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          if (lane == 0) bulk_wait_read_0();  // the previous store has read the box
          __syncwarp();
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t r[32];
            tmem_ld32_sync(tmem_base + lane_off + colO + uint32_t(half * 64 + c * 32), r);
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float lo, hi;
              f32x2_split(mul_f32x2(f32x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), inv_l2), lo,
                          hi);
              w[i] = kStats ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int chunk = c * 4 + q;  // 16-byte chunk of this lane's 128-byte row
              *reinterpret_cast<uint4*>(stg + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                  make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.Mq) {
            tma_store_3d(&omap, stg, it.head * kD + half * 64, row0, it.shard);
            bulk_commit();
          }
        }
        // Statistics mode: each row's log-sum-exp of the scaled scores in log2
        // units, m + log2(l).
        if constexpr (kStats) {
          if (row0 + lane < p.Mq)
            p.lse[(int64_t(it.shard) * p.Hs + it.head) * p.Mq + row0 + lane] = m_run + log2f(l_run);
        }
        tc_fence_before();
      }
    }
    if (!ok && lane == 0) report_timeout(p.err, abort_flag);
    if (lane == 0) bulk_wait_all();  // this warp's TMA stores are complete before the CTA exits
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

cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& a, int num_sms, cudaStream_t s) {
  if (a.Mq <= 0 || a.Mk <= 0) return cudaSuccess;
  // Persistent: one CTA per SM (at most one per work item), each walking the
  // items blockIdx.x, blockIdx.x + gridDim.x, ... so that one item's last
  // blocks and output overlap the next item's Q/K/V loads and first S.
  const int q_blocks = (a.Mq + kTiles * kBQ - 1) / (kTiles * kBQ);
  const int64_t n_items = int64_t(q_blocks) * a.T * a.Hs;
  const int64_t grid = n_items < num_sms ? n_items : num_sms;
  const auto kernel = a.stats ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return note_cuda_error("attention: set shared memory size", e);
  kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, s>>>(maps.q, maps.kv, maps.o, a);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    cudaFuncAttributes fa{};
    char detail[160];
    if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess)
      snprintf(detail, sizeof(detail), "kernel: %d registers/thread, max %d threads/block, %zu B static smem",
               fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes);
    else
      snprintf(detail, sizeof(detail), "kernel attributes unavailable");
    return note_cuda_error("attention: launch", e, detail);
  }
  return cudaSuccess;
}

}  // namespace tp
