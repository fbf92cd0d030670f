// slice.cu - a1, shard slicing: a coalesced 128-bit vectorised blocked copy.
//
// A colwise shard (rows [r*N/T, (r+1)*N/T) of a row-major W[N x K]) is one
// contiguous span; a rowwise shard (columns [r*K/T, (r+1)*K/T) of every row)
// is N row segments of K/T elements at stride K; the packed head split of a
// fused QKV weight is three contiguous spans; a packed block (section "Fused
// projections") is one of these per block, written at the block's offset
// inside the shard (a destination row stride for packed rowwise).  All are
// instances of a blocked 2-D copy, done here with 16-byte loads/stores.  Each
// thread keeps four 16-byte loads in flight before storing, and loads/stores
// use the streaming cache policy: the data is touched exactly once.
#include "internal.h"

namespace tp {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) slice_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                              uint32_t rows, uint32_t c8, int64_t src_ld8,
                                                              int64_t dst_ld8, int64_t src_b8, int64_t dst_b8,
                                                              int64_t src_b8_2, int64_t dst_b8_2) {
  const uint32_t total = rows * c8;  // chunks in this block (host guarantees < 2^31)
  const uint4* s = src + int64_t(blockIdx.y) * src_b8 + int64_t(blockIdx.z) * src_b8_2;
  uint4* d = dst + int64_t(blockIdx.y) * dst_b8 + int64_t(blockIdx.z) * dst_b8_2;
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t base = blockIdx.x * kThreads + threadIdx.x; base < total; base += stride * kUnroll) {
    uint4 v[kUnroll];
    int64_t doff[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t j = base + u * stride;
      if (j < total) {
        const uint32_t r = j / c8;
        const uint32_t c = j - r * c8;
        v[u] = __ldcs(s + int64_t(r) * src_ld8 + c);
        doff[u] = int64_t(r) * dst_ld8 + c;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t j = base + u * stride;
      if (j < total) __stcs(d + doff[u], v[u]);
    }
  }
}

// Several blocked 2-D copies in one launch.  Job j owns CTAs
// [cta0[j], cta0[j+1]) and walks its flattened (block, row, chunk) index
// space with them; a job that is one contiguous span per block has rows = 1
// and a single block needs no division (the branches are uniform per CTA).
struct SliceJobs {
  const uint4* src[kSliceJobsPerLaunch];
  uint4* dst[kSliceJobsPerLaunch];
  uint32_t nblocks[kSliceJobsPerLaunch], rows[kSliceJobsPerLaunch], c8[kSliceJobsPerLaunch];
  int64_t src_ld8[kSliceJobsPerLaunch], dst_ld8[kSliceJobsPerLaunch], src_b8[kSliceJobsPerLaunch], dst_b8[kSliceJobsPerLaunch];
  int cta0[kSliceJobsPerLaunch + 1];
  int njobs;
};

__global__ void __launch_bounds__(kThreads) slice_jobs_kernel(const __grid_constant__ SliceJobs J) {
  int j = 0;
  while (j + 1 < J.njobs && int(blockIdx.x) >= J.cta0[j + 1]) ++j;
  const uint32_t nb = J.nblocks[j], rows = J.rows[j], c8 = J.c8[j];
  const uint32_t per_block = rows * c8;
  const uint32_t total = nb * per_block;  // < 2^31 (host)
  const uint32_t stride = uint32_t(J.cta0[j + 1] - J.cta0[j]) * kThreads;
  const uint4* src = J.src[j];
  uint4* dst = J.dst[j];
  for (uint32_t base = (blockIdx.x - uint32_t(J.cta0[j])) * kThreads + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
    int64_t doff[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t i = base + u * stride;
      if (i < total) {
        uint32_t b = 0, rem = i;
        if (nb > 1) {
          b = i / per_block;
          rem = i - b * per_block;
        }
        uint32_t r = 0, c = rem;
        if (rows > 1) {
          r = rem / c8;
          c = rem - r * c8;
        }
        v[u] = __ldcs(src + int64_t(b) * J.src_b8[j] + int64_t(r) * J.src_ld8[j] + c);
        doff[u] = int64_t(b) * J.dst_b8[j] + int64_t(r) * J.dst_ld8[j] + c;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t i = base + u * stride;
      if (i < total) __stcs(dst + doff[u], v[u]);
    }
  }
}

}  // namespace

cudaError_t launch_slice_jobs(const SliceJob* jobs, int njobs, cudaStream_t st) {
  if (njobs <= 0) return cudaSuccess;
  if (njobs > kSliceJobsPerLaunch) return note_cuda_error("slice jobs: too many jobs", cudaErrorInvalidValue);
  SliceJobs J{};
  int64_t chunks[kSliceJobsPerLaunch], all = 0;
  bool fits = true;
  for (int j = 0; j < njobs; ++j) {
    SliceJob s = jobs[j];
    if (s.src_ld == s.cols && s.dst_ld == s.cols) {  // contiguous per block: one long row
      s.cols *= s.rows;
      s.rows = 1;
      s.src_ld = s.dst_ld = s.cols;
    }
    chunks[j] = s.nblocks * s.rows * (s.cols / 8);
    if (chunks[j] >= (int64_t(1) << 31) - int64_t(kThreads) * kUnroll * 148 * 16) fits = false;
    J.src[j] = reinterpret_cast<const uint4*>(s.src);
    J.dst[j] = reinterpret_cast<uint4*>(s.dst);
    J.nblocks[j] = uint32_t(s.nblocks);
    J.rows[j] = uint32_t(s.rows);
    J.c8[j] = uint32_t(s.cols / 8);
    J.src_ld8[j] = s.src_ld / 8;
    J.dst_ld8[j] = s.dst_ld / 8;
    J.src_b8[j] = s.src_bstride / 8;
    J.dst_b8[j] = s.dst_bstride / 8;
    all += chunks[j];
  }
  if (!fits) {  // a job too large for 32-bit indexing: one launch per job
    for (int j = 0; j < njobs; ++j) {
      const SliceJob& s = jobs[j];
      cudaError_t e = launch_slice_copy(s.src, s.dst, s.nblocks, s.rows, s.cols, s.src_ld, s.src_bstride,
                                        s.dst_bstride, st, 1, 0, 0, s.dst_ld);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (all == 0) return cudaSuccess;
  // CTAs in proportion to each job's bytes (at least one each), about 16 per SM in all.
  const int64_t budget = 148 * 16;
  int cta = 0;
  for (int j = 0; j < njobs; ++j) {
    J.cta0[j] = cta;
    int64_t n = (chunks[j] * budget + all - 1) / all;
    const int64_t need = (chunks[j] + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    if (n > need) n = need;
    if (n < 1) n = 1;
    cta += int(n);
  }
  J.cta0[njobs] = cta;
  J.njobs = njobs;
  slice_jobs_kernel<<<cta, kThreads, 0, st>>>(J);
  count_launch();
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? e : note_cuda_error("slice jobs: launch", e);
}

cudaError_t launch_slice_copy(const uint16_t* src, uint16_t* dst, int64_t nblocks, int64_t rows, int64_t cols,
                              int64_t src_ld, int64_t src_bstride, int64_t dst_bstride, cudaStream_t st,
                              int64_t nblocks2, int64_t src_bstride2, int64_t dst_bstride2, int64_t dst_ld) {
  if (nblocks <= 0 || nblocks2 <= 0 || rows <= 0 || cols <= 0) return cudaSuccess;
  if (dst_ld < 0) dst_ld = cols;
  // A contiguous copy (row segments back to back on both sides) is one long
  // span, split into virtual rows so the 32-bit chunk index never overflows.
  if (src_ld == cols && dst_ld == cols) {
    int64_t n8 = rows * cols / 8;
    int64_t vc8 = 1;
    for (int64_t cand : {int64_t(4096), int64_t(1024), int64_t(256), int64_t(64), int64_t(8), int64_t(1)})
      if (n8 % cand == 0) { vc8 = cand; break; }
    rows = n8 / vc8;
    cols = vc8 * 8;
    src_ld = cols;
    dst_ld = cols;
  }
  const int64_t c8 = cols / 8;
  // Split very tall copies into pieces whose chunk count fits 31 bits.
  const int64_t max_rows = (int64_t(1) << 30) / c8;
  for (int64_t r0 = 0; r0 < rows; r0 += max_rows) {
    const int64_t nr = rows - r0 < max_rows ? rows - r0 : max_rows;
    const int64_t total = nr * c8;
    int64_t blocks = (total + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(nblocks), static_cast<unsigned>(nblocks2));
    slice_copy_kernel<<<grid, kThreads, 0, st>>>(reinterpret_cast<const uint4*>(src + r0 * src_ld),
                                                 reinterpret_cast<uint4*>(dst + r0 * dst_ld), uint32_t(nr),
                                                 uint32_t(c8), src_ld / 8, dst_ld / 8, src_bstride / 8,
                                                 dst_bstride / 8, src_bstride2 / 8, dst_bstride2 / 8);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return note_cuda_error("slice: launch", e);
  }
  return cudaSuccess;
}

}  // namespace tp
