// api.cu - the C ABI declared in include/tp.h: argument checks, workspace
// layout, TMA tensor maps, handles, and the launch sequence of each layer.
//
// Error policy (Diffusers "Tensor parallelism" page, sections "Limitations"
// and "Constraints and validation"): every constraint is checked before any
// weight is sliced or any kernel is launched, and a failed check returns an
// error instead of doing something else silently.  Nothing here computes on
// the host: every step of every layer runs in the kernels of slice.cu,
// gemm.cu, attn.cu and reduce.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/tp.h"
#include "internal.h"
#include "ptx.cuh"

namespace tp {

__device__ int g_device_error;  // OR of kErr* bits set by kernels' bounded waits

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kMlpMagic = 0x54504D4C50484E44ull;   // "TPMLPHND"
constexpr uint64_t kAttnMagic = 0x5450415454484E44ull;  // "TPATTHND"
constexpr uint64_t kJointMagic = 0x54504A4E54484E44ull; // "TPJNTHND"
constexpr int64_t kMaxDim = int64_t(1) << 31;           // TMA coordinates are 32-bit
constexpr int kMaxPackedBlocks = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int* err = nullptr;  // device address of g_device_error
  // A second stream and two events, on which the joint-attention layer runs
  // the text stream's projections beside the image stream's (created at first
  // use; side_mu keeps one caller's fork/join sequence together).
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex side_mu;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
std::atomic<uint64_t> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

tp_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TP_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return TP_ERR_CUDA;
    d.err = static_cast<int*>(p);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return TP_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return TP_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t n) { return (n + 255) & ~size_t(255); }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int mlp_shape_status(int64_t M, int64_t D, int64_t F, int T) {
  if (T < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || D < 1 || F < 1 || M >= kMaxDim || D >= kMaxDim || F >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (F % T != 0) return TP_ERR_INDIVISIBLE;
  if (D % 8 != 0 || (F / T) % 8 != 0) return TP_ERR_ALIGNMENT;
  return TP_OK;
}

thread_local char g_last_error[512] = "";

cudaError_t note_cuda_error(const char* where, cudaError_t e, const char* detail) {
  if (e != cudaSuccess)
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)%s%s", where, cudaGetErrorName(e), cudaGetErrorString(e),
             detail ? "; " : "", detail ? detail : "");
  return e;
}

int current_device_context(int* num_sms, int** err) {
  DeviceInfo* di = nullptr;
  const tp_status st = device_info(&di);
  if (st != TP_OK) return st;
  *num_sms = di->num_sms;
  *err = di->err;
  return TP_OK;
}

static CUresult make_map_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                            uint64_t d2, uint32_t box0, uint32_t box1, uint32_t box2 = 1, uint64_t d1_stride = 0) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * (d1_stride ? d1_stride : d1) * 2};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {box0, box1, box2};
  const cuuint32_t estride[3] = {1, 1, 1};
  return g_encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                          uint32_t box1, uint64_t d1_stride) {
  return make_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d0, d1, d2, box0, box1, 1, d1_stride);
}

CUresult make_map_3d_bf16_box(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t box0, uint32_t box1, uint32_t box2) {
  return make_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d0, d1, d2, box0, box1, box2);
}

CUresult make_map_out_u16(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t g, uint64_t row_stride,
                          uint64_t group_stride) {
  const cuuint64_t dims[3] = {n, m, g};
  const cuuint64_t strides[2] = {row_stride * 2, (group_stride ? group_stride : row_stride * m) * 2};
  const cuuint32_t box[3] = {64, 32, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, base, dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_map_out_f32(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t g, uint64_t row_stride,
                          uint64_t group_stride) {
  const cuuint64_t dims[3] = {n, m, g};
  const cuuint64_t strides[2] = {row_stride * 4, (group_stride ? group_stride : row_stride * m) * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_map_3d_f16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box0,
                         uint32_t box1) {
  return make_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, d0, d1, d2, box0, box1);
}

namespace {

// ---------------------------------------------------------------------------
// Internal launch helpers (arguments already validated).
// ---------------------------------------------------------------------------

// colwise: out[g] = epi(X . W[g]^T + b[g]), g < T.
// out_rows: rows of each group's output block (0 = M; larger when `out` is a
// row range of a taller [T][out_rows][Ns] buffer).
tp_status run_colwise(DeviceInfo* di, const uint16_t* X, int64_t M, int64_t K, const uint16_t* W, const uint16_t* b,
                      int64_t Ns, int T, int gelu, int out_f16, uint16_t* out, cudaStream_t s, int64_t out_rows = 0,
                      int sms = 0) {
  if (M == 0) return TP_OK;
  const GemmOperand A{X, uint64_t(K), uint64_t(M), 1};
  const GemmOperand B{W, uint64_t(K), uint64_t(Ns), uint64_t(T)};
  GemmArgs a{};
  a.M = int(M);
  a.N = int(Ns);
  a.k_blocks = int((K + 63) / 64);
  a.kshards = 1;
  a.groups = T;
  a.a_follows_shard = 0;
  a.out = out;
  a.out_gstride = (out_rows ? out_rows : M) * Ns;
  a.ldo = Ns;
  a.bias = b;
  a.bias_gstride = Ns;
  a.gelu = gelu;
  a.out_f16 = out_f16;
  a.err = di->err;
  return launch_gemm(A, B, a, sms > 0 ? sms : di->num_sms, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// rowwise: Y = sum_r A[r] . W[r]^T + bias.  a_rows: rows of each shard's A
// block in memory (0 = M; larger when A is a row range of a taller buffer).
tp_status run_rowwise(DeviceInfo* di, const uint16_t* A, int64_t M, int64_t Ks, const uint16_t* W, int64_t N,
                      const uint16_t* bias, int T, void* Y, cudaStream_t s, int64_t a_rows = 0, bool out_f32 = false,
                      int sms = 0) {
  if (M == 0) return TP_OK;
  const GemmOperand Aop{A, uint64_t(Ks), uint64_t(M), uint64_t(T), uint64_t(a_rows)};
  const GemmOperand Bop{W, uint64_t(Ks), uint64_t(N), uint64_t(T)};
  GemmArgs a{};
  a.M = int(M);
  a.N = int(N);
  a.k_blocks = int((Ks + 63) / 64);
  a.kshards = T;
  a.groups = 1;
  a.a_follows_shard = 1;
  a.out = Y;
  a.out_gstride = 0;
  a.ldo = N;
  a.bias = bias;
  a.bias_gstride = 0;
  a.gelu = 0;
  a.out_f16 = 0;
  a.out_f32 = out_f32 ? 1 : 0;
  a.err = di->err;
  return launch_gemm(Aop, Bop, a, sms > 0 ? sms : di->num_sms, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// SwiGLU colwise: out[g] = silu(X W_gate,g^T + bg) * (X W_up,g^T + bu), W[g] = [gate; up].
tp_status run_colwise_swiglu(DeviceInfo* di, const uint16_t* X, int64_t M, int64_t K, const uint16_t* W,
                             const uint16_t* b, int64_t Fs, int T, uint16_t* out, cudaStream_t s) {
  if (M == 0) return TP_OK;
  const GemmOperand A{X, uint64_t(K), uint64_t(M), 1};
  const GemmOperand B{W, uint64_t(K), uint64_t(2 * Fs), uint64_t(T)};
  GemmArgs a{};
  a.M = int(M);
  a.N = int(Fs);
  a.k_blocks = int((K + 63) / 64);
  a.kshards = 1;
  a.groups = T;
  a.out = out;
  a.out_gstride = M * Fs;
  a.ldo = Fs;
  a.bias = b;
  a.bias_gstride = 2 * Fs;
  a.swiglu = 1;
  a.up_off = Fs;
  a.err = di->err;
  return launch_gemm(A, B, a, di->num_sms, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// rowwise_split_input: Y = sum_r X[:, r*Ks:(r+1)*Ks] . W[r]^T + bias, X read in place.
tp_status run_rowwise_split(DeviceInfo* di, const uint16_t* X, int64_t M, int64_t Ks, const uint16_t* W, int64_t N,
                            const uint16_t* bias, int T, uint16_t* Y, cudaStream_t s) {
  if (M == 0) return TP_OK;
  const GemmOperand Aop{X, uint64_t(Ks), uint64_t(M), uint64_t(T)};  // memory [M][T][Ks]
  const GemmOperand Bop{W, uint64_t(Ks), uint64_t(N), uint64_t(T)};
  GemmArgs a{};
  a.M = int(M);
  a.N = int(N);
  a.k_blocks = int((Ks + 63) / 64);
  a.kshards = T;
  a.groups = 1;
  a.a_split_input = 1;
  a.out = Y;
  a.ldo = N;
  a.bias = bias;
  a.err = di->err;
  return launch_gemm(Aop, Bop, a, di->num_sms, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// Per-shard SDPA.  Queries: the Q columns of Qsrc [T][Mq][3*Hs*128]; keys and
// values: the K and V columns of KVsrc [T][Mk][3*Hs*128] (the same buffer for
// ordinary attention).  Output: bf16 O [T][Mq][Hs*128], or in the statistics
// mode fp16 O and fp32 lse [T][Hs][Mq].
tp_status run_sdpa_qkv(DeviceInfo* di, const uint16_t* Qsrc, int64_t Mq, const uint16_t* KVsrc, int64_t Mk, int Hs,
                       int T, void* O, bool stats, float* lse, cudaStream_t s) {
  if (Mq == 0 || Mk == 0) return TP_OK;
  const uint64_t cols = uint64_t(3) * Hs * TP_HEAD_DIM;
  AttnMaps m;
  const CUresult om =
      make_map_out_u16(&m.o, O, uint64_t(Hs) * TP_HEAD_DIM, uint64_t(Mq), uint64_t(T), uint64_t(Hs) * TP_HEAD_DIM, 0);
  if (make_map_3d_f16(&m.q, Qsrc, cols, uint64_t(Mq), uint64_t(T), 64, 128) != CUDA_SUCCESS ||
      make_map_3d_f16(&m.kv, KVsrc, cols, uint64_t(Mk), uint64_t(T), 64, 128) != CUDA_SUCCESS || om != CUDA_SUCCESS) {
    note_cuda_error("attention: tensor map encode", cudaErrorInvalidValue);
    return TP_ERR_CUDA;
  }
  AttnArgs a{};
  a.Mq = int(Mq);
  a.Mk = int(Mk);
  a.Hs = Hs;
  a.T = T;
  a.q_col0 = 0;
  a.k_col0 = Hs * TP_HEAD_DIM;
  a.v_col0 = 2 * Hs * TP_HEAD_DIM;
  a.stats = stats ? 1 : 0;
  a.lse = lse;
  a.scale_log2 = float(1.4426950408889634 / std::sqrt(double(TP_HEAD_DIM)));  // log2(e) / sqrt(d)
  a.err = di->err;
  return launch_attention(m, a, di->num_sms, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status run_sdpa(DeviceInfo* di, const uint16_t* QKV, int64_t M, int heads, int T, uint16_t* O, cudaStream_t s) {
  return run_sdpa_qkv(di, QKV, M, QKV, M, heads / T, T, O, false, nullptr, s);
}

// Slices of whole weights (all T shards), used by the one-shot calls and prepare.
tp_status slice_all_colwise(const uint16_t* W, int64_t rows, int64_t cols, uint16_t* out, cudaStream_t s) {
  // Colwise shards stacked in rank order occupy W's own layout: one contiguous copy.
  return launch_slice_copy(W, out, 1, rows, cols, cols, 0, 0, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status slice_all_rowwise(const uint16_t* W, int64_t rows, int64_t cols, int T, uint16_t* out, cudaStream_t s) {
  const int64_t cs = cols / T;
  // shard r: rows x cs block starting at column r*cs; blocks are the shards.
  return launch_slice_copy(W, out, T, rows, cs, cols, cs, rows * cs, s) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// Job builders for batched slicing (one launch for a layer's weights).
// All colwise shards of W[rows x cols] stacked: the weight's own bytes.
SliceJob job_colwise_all(const uint16_t* W, int64_t rows, int64_t cols, uint16_t* out) {
  return SliceJob{W, out, 1, rows, cols, cols, cols, 0, 0};
}
// All rowwise shards: block r = columns [r*cols/T, (r+1)*cols/T) of every row.
SliceJob job_rowwise_all(const uint16_t* W, int64_t rows, int64_t cols, int T, uint16_t* out) {
  const int64_t cs = cols / T;
  return SliceJob{W, out, T, rows, cs, cols, cs, cs, rows * cs};
}
// Head split of a fused [Q; K; V] weight (packed colwise, blocks [1, 1, 1]):
// three jobs, block x of shard r from rows x*D + r*D/T to out rows (3r + x)*D/T.
void jobs_qkv_all(const uint16_t* Wqkv, int64_t D, int T, uint16_t* out, SliceJob* jobs) {
  const int64_t rs = D / T;
  for (int x = 0; x < 3; ++x) jobs[x] = SliceJob{Wqkv + x * D * D, out + x * rs * D, T, rs, D, D, D, rs * D, 3 * rs * D};
}

tp_status slice_all_qkv(const uint16_t* Wqkv, int64_t D, int T, uint16_t* out, cudaStream_t s) {
  // shard r = [Q_r; K_r; V_r]; X_r = rows [r*D/T, (r+1)*D/T) of block X.  One
  // launch: block (r, x) copies X_r from Wqkv[x*D + r*D/T] to out[(3r + x)*D/T].
  const int64_t rs = D / T;
  return launch_slice_copy(Wqkv, out, T, rs, D, D, rs * D, 3 * rs * D, s, 3, D * D, rs * D) == cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

// Packed slicing ("Fused projections") as blocked copies: one SliceJob per
// packed block, covering every shard (rank < 0) or one shard.  sizes[] are
// absolute block sizes along the packed dimension (validated).  Returns the
// number of jobs written to `out_jobs`.
int packed_jobs(const uint16_t* W, int64_t rows, int64_t cols, int style, const int64_t* sizes, int nb, int T,
                int rank, uint16_t* out, SliceJob* out_jobs) {
  const int64_t P = style == TP_COLWISE ? rows : cols;
  const int64_t Ps = P / T;  // shard extent along the packed dimension
  int64_t start = 0, off = 0;
  for (int b = 0; b < nb; ++b) {
    const int64_t q = sizes[b] / T;  // this block's share per shard
    const int64_t r0 = rank < 0 ? 0 : rank;
    const int64_t nblk = rank < 0 ? T : 1;
    if (style == TP_COLWISE)
      out_jobs[b] = SliceJob{W + (start + r0 * q) * cols, out + off * cols, nblk, q, cols, cols, cols, q * cols,
                             Ps * cols};
    else
      out_jobs[b] = SliceJob{W + start + r0 * q, out + off, nblk, rows, q, cols, Ps, q, rows * Ps};
    start += sizes[b];
    off += q;
  }
  return nb;
}

// Launches jobs in groups of kSliceJobsPerLaunch.
tp_status run_slice_jobs(const SliceJob* jobs, int n, cudaStream_t s) {
  for (int i = 0; i < n; i += kSliceJobsPerLaunch) {
    const int k = n - i < kSliceJobsPerLaunch ? n - i : kSliceJobsPerLaunch;
    if (launch_slice_jobs(jobs + i, k, s) != cudaSuccess) return TP_ERR_CUDA;
  }
  return TP_OK;
}

tp_status slice_packed(const uint16_t* W, int64_t rows, int64_t cols, int style, const int64_t* sizes, int nb,
                       int T, int rank, uint16_t* out, cudaStream_t s) {
  SliceJob jobs[kMaxPackedBlocks];
  const int n = packed_jobs(W, rows, cols, style, sizes, nb, T, rank, out, jobs);
  return run_slice_jobs(jobs, n, s);
}

// Validates a packed call and turns proportional blocks into absolute sizes.
tp_status check_packed(const uint16_t* W, int64_t rows, int64_t cols, int style, const int64_t* blocks, int nblocks,
                       int T, const uint16_t* out, int64_t* sizes) {
  if (!W || !out || !blocks) return TP_ERR_NULL;
  if (style != TP_COLWISE && style != TP_ROWWISE) return TP_ERR_BAD_STYLE;
  if (T < 1) return TP_ERR_BAD_DEGREE;
  if (rows < 1 || cols < 1 || rows >= kMaxDim || cols >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (nblocks < 1 || nblocks > kMaxPackedBlocks) return TP_ERR_BAD_BLOCKS;
  const int64_t P = style == TP_COLWISE ? rows : cols;
  int64_t sum = 0;
  for (int b = 0; b < nblocks; ++b) {
    if (blocks[b] < 1 || blocks[b] > P) return TP_ERR_BAD_BLOCKS;
    sum += blocks[b];
  }
  if (sum > P || P % sum != 0) return TP_ERR_BAD_BLOCKS;
  for (int b = 0; b < nblocks; ++b) {
    sizes[b] = blocks[b] * (P / sum);
    if (sizes[b] % T != 0) return TP_ERR_INDIVISIBLE;
  }
  if (!al16(W) || !al16(out) || cols % 8 != 0) return TP_ERR_ALIGNMENT;
  if (style == TP_ROWWISE)
    for (int b = 0; b < nblocks; ++b)
      if ((sizes[b] / T) % 8 != 0) return TP_ERR_ALIGNMENT;
  return TP_OK;
}

// ---------------------------------------------------------------------------
// Shape checks shared by the layer calls.
// ---------------------------------------------------------------------------
tp_status check_mlp_shape(int64_t M, int64_t D, int64_t F, int T) {
  return tp_status(mlp_shape_status(M, D, F, T));
}

tp_status check_attn_shape(int64_t M, int64_t D, int heads, int T) {
  if (T < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || D < 1 || heads < 1 || M >= kMaxDim || D >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (heads % T != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (D != int64_t(heads) * TP_HEAD_DIM) return TP_ERR_BAD_SHAPE;
  return TP_OK;
}

struct MlpLayout {
  size_t w_up, b_up, w_down, h, total;
};
// swiglu: the colwise weight is [gate; up], twice the rows of W_up.
MlpLayout mlp_layout(int64_t M, int64_t D, int64_t F, bool with_weights, bool swiglu = false) {
  MlpLayout L{};
  size_t off = 0;
  const size_t in_rows = size_t(F) * (swiglu ? 2 : 1);
  if (with_weights) {
    L.w_up = off;
    off += up256(in_rows * D * 2);
    L.b_up = off;
    off += up256(in_rows * 2);
    L.w_down = off;
    off += up256(size_t(D) * F * 2);
  }
  L.h = off;
  off += up256(size_t(M) * F * 2);
  L.total = off;
  return L;
}

struct AttnLayout {
  size_t w_qkv, w_o, qkv, o, total;
};
AttnLayout attn_layout(int64_t M, int64_t D, bool with_weights) {
  AttnLayout L{};
  size_t off = 0;
  if (with_weights) {
    L.w_qkv = off;
    off += up256(size_t(3) * D * D * 2);
    L.w_o = off;
    off += up256(size_t(D) * D * 2);
  }
  L.qkv = off;
  off += up256(size_t(M) * 3 * D * 2);
  L.o = off;
  off += up256(size_t(M) * D * 2);
  L.total = off;
  return L;
}

tp_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return TP_OK;
  if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return TP_ERR_WORKSPACE;
  return TP_OK;
}

// The MLP pair on sharded weights (a2..a4); swiglu: w_up_sh holds [gate_r; up_r].
tp_status mlp_forward(DeviceInfo* di, const uint16_t* X, int64_t M, int64_t D, int64_t F, int T,
                      const uint16_t* w_up_sh, const uint16_t* b_up_sh, const uint16_t* w_down_sh,
                      const uint16_t* b_down, uint16_t* H, uint16_t* Y, cudaStream_t s, bool swiglu = false) {
  const int64_t Fs = F / T;
  tp_status st = swiglu ? run_colwise_swiglu(di, X, M, D, w_up_sh, b_up_sh, Fs, T, H, s)
                        : run_colwise(di, X, M, D, w_up_sh, b_up_sh, Fs, T, 1, 0, H, s);
  if (st != TP_OK) return st;
  return run_rowwise(di, H, M, Fs, w_down_sh, D, b_down, T, Y, s);
}

// The attention block on sharded weights (a5..a7).
tp_status attn_forward(DeviceInfo* di, const uint16_t* X, int64_t M, int64_t D, int heads, int T,
                       const uint16_t* w_qkv_sh, const uint16_t* w_o_sh, uint16_t* QKV, uint16_t* O, uint16_t* Y,
                       cudaStream_t s) {
  const int64_t Ds = D / T;
  // Q/K/V are stored in fp16 for the attention kernel (see attn.cu, "Precision").
  tp_status st = run_colwise(di, X, M, D, w_qkv_sh, nullptr, 3 * Ds, T, 0, 1, QKV, s);
  if (st != TP_OK) return st;
  st = run_sdpa(di, QKV, M, heads, T, O, s);
  if (st != TP_OK) return st;
  return run_rowwise(di, O, M, Ds, w_o_sh, D, nullptr, T, Y, s);
}

// Dual-stream joint attention on sharded weights: both streams' head-split
// QKV land in one [T][Mi+Mt][3*Ds] buffer (image rows first), one SDPA runs
// over the joint tokens, and each stream's rows of O go through its own
// rowwise out-projection (read in place as a row range of O).
//
// The two streams' projections are independent, so when both have tokens the
// text stream's GEMM runs on a side stream over a share of the SMs in
// proportion to its rows, beside the image stream's GEMM on the rest: the
// short text launch no longer runs alone on a partly idle GPU.  Each GEMM's
// per-element arithmetic does not depend on its SM budget, so the outputs are
// the same as with the two launches in sequence.
tp_status joint_attn_forward(DeviceInfo* di, const uint16_t* X_img, int64_t Mi, const uint16_t* X_txt, int64_t Mt,
                             int64_t D, int heads, int T, const uint16_t* wq_img, const uint16_t* wq_txt,
                             const uint16_t* wo_img, const uint16_t* wo_txt, uint16_t* QKV, uint16_t* O,
                             uint16_t* Y_img, uint16_t* Y_txt, cudaStream_t s) {
  const int64_t Ds = D / T, M = Mi + Mt;
  uint16_t* qkv_txt = QKV + Mi * 3 * Ds;
  const uint16_t* o_txt = O + Mi * Ds;
  if (Mi == 0 || Mt == 0 || di->num_sms < 8) {
    tp_status st = run_colwise(di, X_img, Mi, D, wq_img, nullptr, 3 * Ds, T, 0, 1, QKV, s, M);
    if (st == TP_OK) st = run_colwise(di, X_txt, Mt, D, wq_txt, nullptr, 3 * Ds, T, 0, 1, qkv_txt, s, M);
    if (st == TP_OK) st = run_sdpa(di, QKV, M, heads, T, O, s);
    if (st == TP_OK) st = run_rowwise(di, O, Mi, Ds, wo_img, D, nullptr, T, Y_img, s, M);
    if (st == TP_OK) st = run_rowwise(di, o_txt, Mt, Ds, wo_txt, D, nullptr, T, Y_txt, s, M);
    return st;
  }
  std::lock_guard<std::mutex> lock(di->side_mu);
  if (di->side == nullptr) {
    cudaError_t e = cudaStreamCreateWithFlags(&di->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&di->fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&di->join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      note_cuda_error("joint attention: side stream", e);
      return TP_ERR_CUDA;
    }
  }
  // SMs for the text stream: its share of the rows, in whole CTA pairs, and
  // at least one pair on each side.
  const int pairs = di->num_sms / 2;
  int txt_pairs = int((int64_t(pairs) * Mt + M / 2) / M);
  if (txt_pairs < 1) txt_pairs = 1;
  if (txt_pairs > pairs - 1) txt_pairs = pairs - 1;
  const int sms_txt = 2 * txt_pairs, sms_img = di->num_sms - sms_txt;
  // Runs img(s) and txt(side) between a fork of `s` and a join back into it;
  // the join is enqueued whatever happened, so `s` never runs ahead of work
  // left on the side stream.
  auto beside = [&](auto img, auto txt) {
    cudaError_t e = cudaEventRecord(di->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(di->side, di->fork, 0);
    if (e != cudaSuccess) {
      note_cuda_error("joint attention: fork", e);
      return TP_ERR_CUDA;
    }
    tp_status st = txt();
    const tp_status si = img();
    if (st == TP_OK) st = si;
    e = cudaEventRecord(di->join, di->side);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, di->join, 0);
    if (e != cudaSuccess) {
      note_cuda_error("joint attention: join", e);
      return TP_ERR_CUDA;
    }
    return st;
  };
  tp_status st = beside(
      [&] { return run_colwise(di, X_img, Mi, D, wq_img, nullptr, 3 * Ds, T, 0, 1, QKV, s, M, sms_img); },
      [&] { return run_colwise(di, X_txt, Mt, D, wq_txt, nullptr, 3 * Ds, T, 0, 1, qkv_txt, di->side, M, sms_txt); });
  if (st == TP_OK) st = run_sdpa(di, QKV, M, heads, T, O, s);
  if (st == TP_OK)
    st = beside(
        [&] { return run_rowwise(di, O, Mi, Ds, wo_img, D, nullptr, T, Y_img, s, M, false, sms_img); },
        [&] { return run_rowwise(di, o_txt, Mt, Ds, wo_txt, D, nullptr, T, Y_txt, di->side, M, false, sms_txt); });
  return st;
}

struct MlpHandle {
  uint64_t magic;
  int device;
  int64_t D, F;
  int T;
  bool swiglu;       // colwise weight holds [gate_r; up_r] per shard
  uint16_t* w_up;    // [T][F/T][D], SwiGLU: [T][2F/T][D]
  uint16_t* b_up;    // [T][F/T] or null, SwiGLU: [T][2F/T]
  uint16_t* w_down;  // [T][D][F/T]
  uint16_t* b_down;  // [D] or null (replicated)
};

struct AttnHandle {
  uint64_t magic;
  int device;
  int64_t D;
  int heads, T;
  uint16_t* w_qkv;  // [T][3D/T][D]
  uint16_t* w_o;    // [T][D][D/T]
};

struct JointHandle {
  uint64_t magic;
  int device;
  int64_t D;
  int heads, T;
  uint16_t* w_qkv_img;  // [T][3D/T][D]
  uint16_t* w_qkv_txt;
  uint16_t* w_o_img;    // [T][D][D/T]
  uint16_t* w_o_txt;
};

struct JointLayout {
  size_t w_qkv_img, w_qkv_txt, w_o_img, w_o_txt, qkv, o, total;
};
JointLayout joint_layout(int64_t M, int64_t D, bool with_weights) {
  JointLayout L{};
  size_t off = 0;
  if (with_weights) {
    const size_t wq = up256(size_t(3) * D * D * 2), wo = up256(size_t(D) * D * 2);
    L.w_qkv_img = off;
    off += wq;
    L.w_qkv_txt = off;
    off += wq;
    L.w_o_img = off;
    off += wo;
    L.w_o_txt = off;
    off += wo;
  }
  L.qkv = off;
  off += up256(size_t(M) * 3 * D * 2);
  L.o = off;
  off += up256(size_t(M) * D * 2);
  L.total = off;
  return L;
}

tp_status check_joint_shape(int64_t Mi, int64_t Mt, int64_t D, int heads, int T) {
  if (Mi < 0 || Mt < 0) return TP_ERR_BAD_SHAPE;
  return check_attn_shape(Mi + Mt, D, heads, T);
}

// One rank's workspaces: the MLP's hidden shard H_r [M x F/T] (bf16); the
// attention's QKV_r [M x 3D/T] (fp16) and O_r [M x D/T] (bf16).
size_t mlp_rank_ws(int64_t M, int64_t F, int T) { return up256(size_t(M) * (F / T) * 2); }
struct AttnRankLayout {
  size_t qkv, o, total;
};
AttnRankLayout attn_rank_layout(int64_t M, int64_t D, int T) {
  AttnRankLayout L{};
  L.qkv = 0;
  L.o = up256(size_t(M) * 3 * (D / T) * 2);
  L.total = L.o + up256(size_t(M) * (D / T) * 2);
  return L;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" {

const char* tp_status_string(int s) {
  switch (s) {
    case TP_OK: return "ok";
    case TP_ERR_NULL: return "a required pointer is NULL";
    case TP_ERR_BAD_DEGREE: return "tp_degree must be >= 1";
    case TP_ERR_BAD_RANK: return "rank outside [0, tp_degree)";
    case TP_ERR_INDIVISIBLE: return "a sharded dimension is not divisible by tp_degree";
    case TP_ERR_HEADS_INDIVISIBLE: return "tp_degree does not divide the number of attention heads";
    case TP_ERR_BAD_SHAPE: return "unsupported shape";
    case TP_ERR_ALIGNMENT: return "pointer or shard row not 16-byte aligned";
    case TP_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case TP_ERR_CUDA: return "CUDA call failed";
    case TP_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait timed out";
    case TP_ERR_BAD_STYLE: return "unknown sharding style";
    case TP_ERR_BAD_HANDLE: return "invalid handle";
    case TP_ERR_BAD_BLOCKS:
      return "packed blocks invalid: count outside 1..64, a block < 1, or their sum does not divide the packed "
             "dimension";
    case TP_ERR_RANGE:
      return "an fp16 activation (Q/K/V) was outside the fp16 range or NaN; the call's output is not valid";
    case TP_ERR_SCRATCH_LIMIT:
      return "size exceeds the 64 MiB static scratch of tp_mlp_pair_sharded_noalloc (F * 256 bytes must fit)";
    default: return "unknown status";
  }
}

int tp_abi_version(void) { return TP_ABI_VERSION; }

const char* tp_last_error_message(void) { return g_last_error; }

uint64_t tp_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

tp_status tp_check_device_error(void* stream) {
  DeviceInfo* di = nullptr;
  tp_status st = device_info(&di);
  if (st != TP_OK) return st;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return TP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, di->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TP_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(di->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TP_ERR_CUDA;
    return (v & kErrTimeout) ? TP_ERR_DEVICE_TIMEOUT : TP_ERR_RANGE;
  }
  return TP_OK;
}

// ----------------------------------------------------------------------- a1
tp_status tp_shard_weight(const uint16_t* W, int64_t rows, int64_t cols, int style, int tp_degree, int rank,
                          uint16_t* out, void* stream) {
  if (!W || !out) return TP_ERR_NULL;
  if (style == TP_ROWWISE_SPLIT_INPUT) style = TP_ROWWISE;  // same weight slice
  if (style != TP_COLWISE && style != TP_ROWWISE) return TP_ERR_BAD_STYLE;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (rank < 0 || rank >= tp_degree) return TP_ERR_BAD_RANK;
  if (rows < 1 || cols < 1) return TP_ERR_BAD_SHAPE;
  if (style == TP_COLWISE && rows % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  if (style == TP_ROWWISE && cols % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  if (!al16(W) || !al16(out) || cols % 8 != 0) return TP_ERR_ALIGNMENT;
  if (style == TP_ROWWISE && (cols / tp_degree) % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaError_t e;
  if (style == TP_COLWISE) {
    const int64_t rs = rows / tp_degree;
    e = launch_slice_copy(W + int64_t(rank) * rs * cols, out, 1, rs, cols, cols, 0, 0, as_stream(stream));
  } else {
    const int64_t cs = cols / tp_degree;
    e = launch_slice_copy(W + int64_t(rank) * cs, out, 1, rows, cs, cols, 0, 0, as_stream(stream));
  }
  return e == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

tp_status tp_shard_weight_all(const uint16_t* W, int64_t rows, int64_t cols, int style, int tp_degree, uint16_t* out,
                              void* stream) {
  if (!W || !out) return TP_ERR_NULL;
  if (style == TP_ROWWISE_SPLIT_INPUT) style = TP_ROWWISE;  // same weight slice
  if (style != TP_COLWISE && style != TP_ROWWISE) return TP_ERR_BAD_STYLE;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (rows < 1 || cols < 1) return TP_ERR_BAD_SHAPE;
  if (style == TP_COLWISE && rows % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  if (style == TP_ROWWISE && cols % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  if (!al16(W) || !al16(out) || cols % 8 != 0) return TP_ERR_ALIGNMENT;
  if (style == TP_ROWWISE && (cols / tp_degree) % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return style == TP_COLWISE ? slice_all_colwise(W, rows, cols, out, as_stream(stream))
                             : slice_all_rowwise(W, rows, cols, tp_degree, out, as_stream(stream));
}

tp_status tp_shard_weights_batch(const tp_shard_job* jobs, int njobs, int tp_degree, void* stream) {
  if (!jobs) return TP_ERR_NULL;
  if (njobs < 1 || njobs > kMaxSliceJobs) return TP_ERR_BAD_SHAPE;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  SliceJob sj[kMaxSliceJobs * kMaxPackedBlocks];
  int n = 0;
  for (int j = 0; j < njobs; ++j) {
    const tp_shard_job& b = jobs[j];
    if (b.blocks) {  // packed job
      int64_t sizes[kMaxPackedBlocks];
      const tp_status st = check_packed(b.W, b.rows, b.cols, b.style, b.blocks, b.nblocks, tp_degree, b.out, sizes);
      if (st != TP_OK) return st;
      n += packed_jobs(b.W, b.rows, b.cols, b.style, sizes, b.nblocks, tp_degree, -1, b.out, sj + n);
      continue;
    }
    int style = b.style == TP_ROWWISE_SPLIT_INPUT ? int(TP_ROWWISE) : b.style;
    if (!b.W || !b.out) return TP_ERR_NULL;
    if (style != TP_COLWISE && style != TP_ROWWISE) return TP_ERR_BAD_STYLE;
    if (b.rows < 1 || b.cols < 1 || b.rows >= kMaxDim || b.cols >= kMaxDim) return TP_ERR_BAD_SHAPE;
    if (style == TP_COLWISE && b.rows % tp_degree != 0) return TP_ERR_INDIVISIBLE;
    if (style == TP_ROWWISE && b.cols % tp_degree != 0) return TP_ERR_INDIVISIBLE;
    if (!al16(b.W) || !al16(b.out) || b.cols % 8 != 0) return TP_ERR_ALIGNMENT;
    if (style == TP_ROWWISE && (b.cols / tp_degree) % 8 != 0) return TP_ERR_ALIGNMENT;
    if (style == TP_COLWISE) {  // all colwise shards stacked = the weight's own bytes
      sj[n++] = SliceJob{b.W, b.out, 1, b.rows, b.cols, b.cols, b.cols, 0, 0};
    } else {  // block r = columns [r*cs, (r+1)*cs) of every row
      const int64_t cs = b.cols / tp_degree;
      sj[n++] = SliceJob{b.W, b.out, tp_degree, b.rows, cs, b.cols, cs, cs, b.rows * cs};
    }
  }
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_slice_jobs(sj, n, as_stream(stream));
}

tp_status tp_shard_bias(const uint16_t* b, int64_t n, int tp_degree, int rank, uint16_t* out, void* stream) {
  if (!b || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (rank < 0 || rank >= tp_degree) return TP_ERR_BAD_RANK;
  if (n < 1) return TP_ERR_BAD_SHAPE;
  if (n % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  const int64_t ns = n / tp_degree;
  if (!al16(b) || !al16(out) || ns % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return launch_slice_copy(b + int64_t(rank) * ns, out, 1, 1, ns, ns, 0, 0, as_stream(stream)) == cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_shard_qkv_heads(const uint16_t* W_qkv, int64_t D, int heads, int tp_degree, int rank, uint16_t* out,
                             void* stream) {
  if (!W_qkv || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (rank < 0 || rank >= tp_degree) return TP_ERR_BAD_RANK;
  if (D < 1 || heads < 1) return TP_ERR_BAD_SHAPE;
  if (heads % tp_degree != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (D != int64_t(heads) * TP_HEAD_DIM) return TP_ERR_BAD_SHAPE;
  if (!al16(W_qkv) || !al16(out)) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  const int64_t rs = D / tp_degree;
  return launch_slice_copy(W_qkv + int64_t(rank) * rs * D, out, 3, rs, D, D, D * D, rs * D, as_stream(stream)) ==
                 cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_shard_qkv_heads_all(const uint16_t* W_qkv, int64_t D, int heads, int tp_degree, uint16_t* out,
                                 void* stream) {
  if (!W_qkv || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (D < 1 || heads < 1) return TP_ERR_BAD_SHAPE;
  if (heads % tp_degree != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (D != int64_t(heads) * TP_HEAD_DIM) return TP_ERR_BAD_SHAPE;
  if (!al16(W_qkv) || !al16(out)) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return slice_all_qkv(W_qkv, D, tp_degree, out, as_stream(stream));
}

tp_status tp_shard_packed(const uint16_t* W, int64_t rows, int64_t cols, int style, const int64_t* blocks,
                          int nblocks, int tp_degree, int rank, uint16_t* out, void* stream) {
  int64_t sizes[kMaxPackedBlocks];
  tp_status st = check_packed(W, rows, cols, style, blocks, nblocks, tp_degree, out, sizes);
  if (st != TP_OK) return st;
  if (rank < 0 || rank >= tp_degree) return TP_ERR_BAD_RANK;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return slice_packed(W, rows, cols, style, sizes, nblocks, tp_degree, rank, out, as_stream(stream));
}

tp_status tp_shard_packed_all(const uint16_t* W, int64_t rows, int64_t cols, int style, const int64_t* blocks,
                              int nblocks, int tp_degree, uint16_t* out, void* stream) {
  int64_t sizes[kMaxPackedBlocks];
  tp_status st = check_packed(W, rows, cols, style, blocks, nblocks, tp_degree, out, sizes);
  if (st != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return slice_packed(W, rows, cols, style, sizes, nblocks, tp_degree, -1, out, as_stream(stream));
}

// ----------------------------------------------------------------------- step-level calls
tp_status tp_colwise_linear(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W_shards,
                            const uint16_t* b_shards, int64_t N_s, int tp_degree, int gelu, int out_dtype,
                            uint16_t* out, void* stream) {
  if (!X || !W_shards || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K < 1 || N_s < 1 || M >= kMaxDim || K >= kMaxDim || N_s * tp_degree >= kMaxDim)
    return TP_ERR_BAD_SHAPE;
  if (!al16(X) || !al16(W_shards) || !al16(out) || (b_shards && !al16(b_shards))) return TP_ERR_ALIGNMENT;
  if (K % 8 != 0 || N_s % 8 != 0) return TP_ERR_ALIGNMENT;
  if (out_dtype != TP_OUT_BF16 && out_dtype != TP_OUT_F16) return TP_ERR_BAD_STYLE;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_colwise(di, X, M, K, W_shards, b_shards, N_s, tp_degree, gelu ? 1 : 0, out_dtype == TP_OUT_F16 ? 1 : 0,
                     out, as_stream(stream));
}

tp_status tp_rowwise_linear_sum(const uint16_t* A_shards, int64_t M, int64_t K_s, const uint16_t* W_shards,
                                int64_t N, const uint16_t* bias, int tp_degree, uint16_t* Y, void* stream) {
  if (!A_shards || !W_shards || !Y) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K_s < 1 || N < 1 || M >= kMaxDim || K_s >= kMaxDim || N >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (!al16(A_shards) || !al16(W_shards) || !al16(Y) || (bias && !al16(bias))) return TP_ERR_ALIGNMENT;
  if (K_s % 8 != 0 || N % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_rowwise(di, A_shards, M, K_s, W_shards, N, bias, tp_degree, Y, as_stream(stream));
}

tp_status tp_colwise_linear_rows(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W_shards,
                                 const uint16_t* b_shards, int64_t N_s, int tp_degree, int gelu, int out_dtype,
                                 uint16_t* out, int64_t out_rows, void* stream) {
  if (out_rows < M || out_rows >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (!X || !W_shards || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K < 1 || N_s < 1 || M >= kMaxDim || K >= kMaxDim || N_s * tp_degree >= kMaxDim)
    return TP_ERR_BAD_SHAPE;
  if (!al16(X) || !al16(W_shards) || !al16(out) || (b_shards && !al16(b_shards))) return TP_ERR_ALIGNMENT;
  if (K % 8 != 0 || N_s % 8 != 0) return TP_ERR_ALIGNMENT;
  if (out_dtype != TP_OUT_BF16 && out_dtype != TP_OUT_F16) return TP_ERR_BAD_STYLE;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_colwise(di, X, M, K, W_shards, b_shards, N_s, tp_degree, gelu ? 1 : 0, out_dtype == TP_OUT_F16 ? 1 : 0,
                     out, as_stream(stream), out_rows);
}

tp_status tp_rowwise_linear_sum_rows(const uint16_t* A_shards, int64_t M, int64_t K_s, int64_t a_rows,
                                     const uint16_t* W_shards, int64_t N, const uint16_t* bias, int tp_degree,
                                     uint16_t* Y, void* stream) {
  if (a_rows < M || a_rows >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (!A_shards || !W_shards || !Y) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K_s < 1 || N < 1 || M >= kMaxDim || K_s >= kMaxDim || N >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (!al16(A_shards) || !al16(W_shards) || !al16(Y) || (bias && !al16(bias))) return TP_ERR_ALIGNMENT;
  if (K_s % 8 != 0 || N % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_rowwise(di, A_shards, M, K_s, W_shards, N, bias, tp_degree, Y, as_stream(stream), a_rows);
}

tp_status tp_colwise_swiglu(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W_shards,
                            const uint16_t* b_shards, int64_t F_s, int tp_degree, uint16_t* out, void* stream) {
  if (!X || !W_shards || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K < 1 || F_s < 1 || M >= kMaxDim || K >= kMaxDim || 2 * F_s * tp_degree >= kMaxDim)
    return TP_ERR_BAD_SHAPE;
  if (!al16(X) || !al16(W_shards) || !al16(out) || (b_shards && !al16(b_shards))) return TP_ERR_ALIGNMENT;
  if (K % 8 != 0 || F_s % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_colwise_swiglu(di, X, M, K, W_shards, b_shards, F_s, tp_degree, out, as_stream(stream));
}

tp_status tp_rowwise_split_input_linear(const uint16_t* X, int64_t M, int64_t K, const uint16_t* W_shards, int64_t N,
                                        const uint16_t* bias, int tp_degree, uint16_t* Y, void* stream) {
  if (!X || !W_shards || !Y) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || K < 1 || N < 1 || M >= kMaxDim || K >= kMaxDim || N >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (K % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  if (!al16(X) || !al16(W_shards) || !al16(Y) || (bias && !al16(bias))) return TP_ERR_ALIGNMENT;
  if ((K / tp_degree) % 8 != 0 || N % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_rowwise_split(di, X, M, K / tp_degree, W_shards, N, bias, tp_degree, Y, as_stream(stream));
}

tp_status tp_sdpa_shards(const uint16_t* QKV, int64_t M, int heads, int tp_degree, uint16_t* O, void* stream) {
  if (!QKV || !O) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || heads < 1 || M >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (heads % tp_degree != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (!al16(QKV) || !al16(O)) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_sdpa(di, QKV, M, heads, tp_degree, O, as_stream(stream));
}

tp_status tp_reduce_partials(const float* parts, int64_t M, int64_t N, int tp_degree, const uint16_t* bias,
                             uint16_t* Y, void* stream) {
  if (!parts || !Y) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (M < 0 || N < 1) return TP_ERR_BAD_SHAPE;
  if (!al16(parts) || !al16(Y) || (bias && !al16(bias)) || N % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return launch_reduce_partials(parts, M, N, tp_degree, bias, Y, as_stream(stream)) == cudaSuccess ? TP_OK
                                                                                                   : TP_ERR_CUDA;
}

tp_status tp_debug_watchdog(uint32_t wait_ms, void* stream) {
  if (wait_ms < 1 || wait_ms > 2000) return TP_ERR_BAD_SHAPE;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return launch_watchdog_probe(di->err, uint64_t(wait_ms) * 1000000ull, as_stream(stream)) == cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

int tp_gemm_tile_plan(int64_t M, int64_t N, int groups, int swiglu) {
  if (M < 1 || N < 1 || groups < 1) return -1;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return -1;
  return gemm_tile_plan(M, N, groups, swiglu != 0, di->num_sms);
}

// ----------------------------------------------------------------------- MLP pair
size_t tp_mlp_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree) {
  if (check_mlp_shape(M, D, F, tp_degree) != TP_OK) return 0;
  return mlp_layout(M, D, F, true).total;
}

size_t tp_mlp_run_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree) {
  if (check_mlp_shape(M, D, F, tp_degree) != TP_OK) return 0;
  return mlp_layout(M, D, F, false).total;
}

tp_status tp_mlp_pair(const uint16_t* X, int64_t M, int64_t D, int64_t F, const uint16_t* W_up,
                      const uint16_t* b_up, const uint16_t* W_down, const uint16_t* b_down, int tp_degree,
                      uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !W_up || !W_down || !Y) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(M, D, F, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(W_up) || !al16(W_down) || !al16(Y) || (b_up && !al16(b_up)) || (b_down && !al16(b_down)))
    return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;  // empty input: nothing to compute or write
  const MlpLayout L = mlp_layout(M, D, F, true);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* w_up_sh = reinterpret_cast<uint16_t*>(w + L.w_up);
  uint16_t* b_up_sh = b_up ? reinterpret_cast<uint16_t*>(w + L.b_up) : nullptr;
  uint16_t* w_down_sh = reinterpret_cast<uint16_t*>(w + L.w_down);
  uint16_t* H = reinterpret_cast<uint16_t*>(w + L.h);
  // a1: materialise every shard (what each rank would hold after sharded
  // loading), W_up, b_up and W_down in one launch.
  const int64_t Fs = F / tp_degree;
  SliceJob sj[3] = {{W_up, w_up_sh, 1, F, D, D, D, 0, 0},
                    {W_down, w_down_sh, tp_degree, D, Fs, F, Fs, Fs, D * Fs},
                    {b_up, b_up_sh, 1, 1, F, F, F, 0, 0}};  // used only when b_up is given
  if (launch_slice_jobs(sj, b_up ? 3 : 2, s) != cudaSuccess) return TP_ERR_CUDA;
  // a2..a4
  return mlp_forward(di, X, M, D, F, tp_degree, w_up_sh, b_up_sh, w_down_sh, b_down, H, Y, s);
}

size_t tp_swiglu_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree) {
  if (check_mlp_shape(M, D, F, tp_degree) != TP_OK) return 0;
  return mlp_layout(M, D, F, true, true).total;
}

tp_status tp_swiglu_mlp_pair(const uint16_t* X, int64_t M, int64_t D, int64_t F, const uint16_t* W_in,
                             const uint16_t* b_in, const uint16_t* W_out, const uint16_t* b_out, int tp_degree,
                             uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !W_in || !W_out || !Y) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(M, D, F, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(W_in) || !al16(W_out) || !al16(Y) || (b_in && !al16(b_in)) || (b_out && !al16(b_out)))
    return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  const MlpLayout L = mlp_layout(M, D, F, true, true);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* w_in_sh = reinterpret_cast<uint16_t*>(w + L.w_up);
  uint16_t* b_in_sh = b_in ? reinterpret_cast<uint16_t*>(w + L.b_up) : nullptr;
  uint16_t* w_out_sh = reinterpret_cast<uint16_t*>(w + L.w_down);
  // [gate; up] packed colwise with blocks [1, 1]: shard r = [gate_r; up_r]
  // (block b of shard r at rows b*Fs of the shard); its bias likewise; W_out
  // rowwise.  One launch.
  const int64_t Fs = F / tp_degree;
  SliceJob sj[5] = {{W_in, w_in_sh, tp_degree, Fs, D, D, D, Fs * D, 2 * Fs * D},
                    {W_in + F * D, w_in_sh + Fs * D, tp_degree, Fs, D, D, D, Fs * D, 2 * Fs * D},
                    {W_out, w_out_sh, tp_degree, D, Fs, F, Fs, Fs, D * Fs}};
  if (b_in) {
    sj[3] = SliceJob{b_in, b_in_sh, tp_degree, 1, Fs, Fs, Fs, Fs, 2 * Fs};
    sj[4] = SliceJob{b_in + F, b_in_sh + Fs, tp_degree, 1, Fs, Fs, Fs, Fs, 2 * Fs};
  }
  if (launch_slice_jobs(sj, b_in ? 5 : 3, s) != cudaSuccess) return TP_ERR_CUDA;
  return mlp_forward(di, X, M, D, F, tp_degree, w_in_sh, b_in_sh, w_out_sh, b_out,
                     reinterpret_cast<uint16_t*>(w + L.h), Y, s, true);
}

tp_status tp_swiglu_prepare(const uint16_t* W_in, const uint16_t* b_in, const uint16_t* W_out, const uint16_t* b_out,
                            int64_t D, int64_t F, int tp_degree, void* stream, void** handle) {
  if (!W_in || !W_out || !handle) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(0, D, F, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(W_in) || !al16(W_out) || (b_in && !al16(b_in)) || (b_out && !al16(b_out))) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  MlpHandle* h = new MlpHandle{};
  h->magic = kMlpMagic;
  cudaGetDevice(&h->device);
  h->D = D;
  h->F = F;
  h->T = tp_degree;
  h->swiglu = true;
  const int64_t halves[2] = {F, F};
  bool ok = cudaMalloc(&h->w_up, size_t(2 * F) * D * 2) == cudaSuccess &&
            cudaMalloc(&h->w_down, size_t(D) * F * 2) == cudaSuccess &&
            (!b_in || cudaMalloc(&h->b_up, size_t(2 * F) * 2) == cudaSuccess) &&
            (!b_out || cudaMalloc(&h->b_down, size_t(D) * 2) == cudaSuccess);
  ok = ok && slice_packed(W_in, 2 * F, D, TP_COLWISE, halves, 2, tp_degree, -1, h->w_up, s) == TP_OK &&
       slice_all_rowwise(W_out, D, F, tp_degree, h->w_down, s) == TP_OK &&
       (!b_in || slice_packed(b_in, 1, 2 * F, TP_ROWWISE, halves, 2, tp_degree, -1, h->b_up, s) == TP_OK) &&
       (!b_out || cudaMemcpyAsync(h->b_down, b_out, size_t(D) * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess);
  if (!ok) {
    tp_destroy(h);
    return TP_ERR_CUDA;
  }
  *handle = h;
  return TP_OK;
}

tp_status tp_mlp_prepare(const uint16_t* W_up, const uint16_t* b_up, const uint16_t* W_down, const uint16_t* b_down,
                         int64_t D, int64_t F, int tp_degree, void* stream, void** handle) {
  if (!W_up || !W_down || !handle) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(0, D, F, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(W_up) || !al16(W_down) || (b_up && !al16(b_up)) || (b_down && !al16(b_down))) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  MlpHandle* h = new MlpHandle{};
  h->magic = kMlpMagic;
  cudaGetDevice(&h->device);
  h->D = D;
  h->F = F;
  h->T = tp_degree;
  bool ok = cudaMalloc(&h->w_up, size_t(F) * D * 2) == cudaSuccess &&
            cudaMalloc(&h->w_down, size_t(D) * F * 2) == cudaSuccess &&
            (!b_up || cudaMalloc(&h->b_up, size_t(F) * 2) == cudaSuccess) &&
            (!b_down || cudaMalloc(&h->b_down, size_t(D) * 2) == cudaSuccess);
  if (ok) {
    SliceJob sj[3] = {job_colwise_all(W_up, F, D, h->w_up), job_rowwise_all(W_down, D, F, tp_degree, h->w_down)};
    if (b_up) sj[2] = job_colwise_all(b_up, 1, F, h->b_up);
    ok = run_slice_jobs(sj, b_up ? 3 : 2, s) == TP_OK;
  }
  ok = ok &&
       (!b_down || cudaMemcpyAsync(h->b_down, b_down, size_t(D) * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess);
  if (!ok) {
    tp_destroy(h);
    return TP_ERR_CUDA;
  }
  *handle = h;
  return TP_OK;
}

tp_status tp_mlp_run(void* handle, const uint16_t* X, int64_t M, uint16_t* Y, void* ws, size_t ws_bytes,
                     void* stream) {
  MlpHandle* h = static_cast<MlpHandle*>(handle);
  if (!h) return TP_ERR_BAD_HANDLE;
  if (h->magic != kMlpMagic) return TP_ERR_BAD_HANDLE;
  if (!X || !Y) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(M, h->D, h->F, h->T);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(Y)) return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  const MlpLayout L = mlp_layout(M, h->D, h->F, false);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  uint16_t* H = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + L.h);
  return mlp_forward(di, X, M, h->D, h->F, h->T, h->w_up, h->b_up, h->w_down, h->b_down, H, Y, as_stream(stream),
                     h->swiglu);
}

// ----------------------------------------------------------------------- attention block
size_t tp_attn_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree) {
  if (check_attn_shape(M, D, heads, tp_degree) != TP_OK) return 0;
  return attn_layout(M, D, true).total;
}

size_t tp_attn_run_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree) {
  if (check_attn_shape(M, D, heads, tp_degree) != TP_OK) return 0;
  return attn_layout(M, D, false).total;
}

tp_status tp_attn_block(const uint16_t* X, int64_t M, int64_t D, const uint16_t* W_qkv, const uint16_t* W_o,
                        int heads, int tp_degree, uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !W_qkv || !W_o || !Y) return TP_ERR_NULL;
  tp_status st = check_attn_shape(M, D, heads, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(W_qkv) || !al16(W_o) || !al16(Y)) return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  const AttnLayout L = attn_layout(M, D, true);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* wq = reinterpret_cast<uint16_t*>(w + L.w_qkv);
  uint16_t* wo = reinterpret_cast<uint16_t*>(w + L.w_o);
  SliceJob sj[4];  // W_qkv head split and W_o rowwise, one launch
  jobs_qkv_all(W_qkv, D, tp_degree, wq, sj);
  sj[3] = job_rowwise_all(W_o, D, D, tp_degree, wo);
  if ((st = run_slice_jobs(sj, 4, s)) != TP_OK) return st;
  return attn_forward(di, X, M, D, heads, tp_degree, wq, wo, reinterpret_cast<uint16_t*>(w + L.qkv),
                      reinterpret_cast<uint16_t*>(w + L.o), Y, s);
}

tp_status tp_attn_prepare(const uint16_t* W_qkv, const uint16_t* W_o, int64_t D, int heads, int tp_degree,
                          void* stream, void** handle) {
  if (!W_qkv || !W_o || !handle) return TP_ERR_NULL;
  tp_status st = check_attn_shape(0, D, heads, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(W_qkv) || !al16(W_o)) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  AttnHandle* h = new AttnHandle{};
  h->magic = kAttnMagic;
  cudaGetDevice(&h->device);
  h->D = D;
  h->heads = heads;
  h->T = tp_degree;
  bool ok = cudaMalloc(&h->w_qkv, size_t(3) * D * D * 2) == cudaSuccess &&
            cudaMalloc(&h->w_o, size_t(D) * D * 2) == cudaSuccess;
  if (ok) {
    SliceJob sj[4];
    jobs_qkv_all(W_qkv, D, tp_degree, h->w_qkv, sj);
    sj[3] = job_rowwise_all(W_o, D, D, tp_degree, h->w_o);
    ok = run_slice_jobs(sj, 4, s) == TP_OK;
  }
  if (!ok) {
    tp_destroy(h);
    return TP_ERR_CUDA;
  }
  *handle = h;
  return TP_OK;
}

tp_status tp_attn_run(void* handle, const uint16_t* X, int64_t M, uint16_t* Y, void* ws, size_t ws_bytes,
                      void* stream) {
  AttnHandle* h = static_cast<AttnHandle*>(handle);
  if (!h) return TP_ERR_BAD_HANDLE;
  if (h->magic != kAttnMagic) return TP_ERR_BAD_HANDLE;
  if (!X || !Y) return TP_ERR_NULL;
  tp_status st = check_attn_shape(M, h->D, h->heads, h->T);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(Y)) return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  const AttnLayout L = attn_layout(M, h->D, false);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  uint8_t* w = static_cast<uint8_t*>(ws);
  return attn_forward(di, X, M, h->D, h->heads, h->T, h->w_qkv, h->w_o, reinterpret_cast<uint16_t*>(w + L.qkv),
                      reinterpret_cast<uint16_t*>(w + L.o), Y, as_stream(stream));
}

// ----------------------------------------------------------------------- dual-stream joint attention
size_t tp_joint_attn_workspace_bytes(int64_t M_img, int64_t M_txt, int64_t D, int heads, int tp_degree) {
  if (check_joint_shape(M_img, M_txt, D, heads, tp_degree) != TP_OK) return 0;
  return joint_layout(M_img + M_txt, D, true).total;
}

size_t tp_joint_attn_run_workspace_bytes(int64_t M_img, int64_t M_txt, int64_t D, int heads, int tp_degree) {
  if (check_joint_shape(M_img, M_txt, D, heads, tp_degree) != TP_OK) return 0;
  return joint_layout(M_img + M_txt, D, false).total;
}

tp_status tp_joint_attn_block(const uint16_t* X_img, int64_t M_img, const uint16_t* X_txt, int64_t M_txt, int64_t D,
                              const uint16_t* W_qkv_img, const uint16_t* W_qkv_txt, const uint16_t* W_o_img,
                              const uint16_t* W_o_txt, int heads, int tp_degree, uint16_t* Y_img, uint16_t* Y_txt,
                              void* ws, size_t ws_bytes, void* stream) {
  if (!W_qkv_img || !W_qkv_txt || !W_o_img || !W_o_txt) return TP_ERR_NULL;
  if ((M_img > 0 && (!X_img || !Y_img)) || (M_txt > 0 && (!X_txt || !Y_txt))) return TP_ERR_NULL;
  tp_status st = check_joint_shape(M_img, M_txt, D, heads, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X_img) || !al16(X_txt) || !al16(Y_img) || !al16(Y_txt) || !al16(W_qkv_img) || !al16(W_qkv_txt) ||
      !al16(W_o_img) || !al16(W_o_txt))
    return TP_ERR_ALIGNMENT;
  if (M_img + M_txt == 0) return TP_OK;
  const JointLayout L = joint_layout(M_img + M_txt, D, true);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  auto at = [w](size_t off) { return reinterpret_cast<uint16_t*>(w + off); };
  SliceJob sj[8];  // both streams' head splits and out-projections, one launch
  jobs_qkv_all(W_qkv_img, D, tp_degree, at(L.w_qkv_img), sj);
  jobs_qkv_all(W_qkv_txt, D, tp_degree, at(L.w_qkv_txt), sj + 3);
  sj[6] = job_rowwise_all(W_o_img, D, D, tp_degree, at(L.w_o_img));
  sj[7] = job_rowwise_all(W_o_txt, D, D, tp_degree, at(L.w_o_txt));
  if ((st = run_slice_jobs(sj, 8, s)) != TP_OK) return st;
  return joint_attn_forward(di, X_img, M_img, X_txt, M_txt, D, heads, tp_degree, at(L.w_qkv_img), at(L.w_qkv_txt),
                            at(L.w_o_img), at(L.w_o_txt), at(L.qkv), at(L.o), Y_img, Y_txt, s);
}

tp_status tp_joint_attn_prepare(const uint16_t* W_qkv_img, const uint16_t* W_qkv_txt, const uint16_t* W_o_img,
                                const uint16_t* W_o_txt, int64_t D, int heads, int tp_degree, void* stream,
                                void** handle) {
  if (!W_qkv_img || !W_qkv_txt || !W_o_img || !W_o_txt || !handle) return TP_ERR_NULL;
  tp_status st = check_attn_shape(0, D, heads, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(W_qkv_img) || !al16(W_qkv_txt) || !al16(W_o_img) || !al16(W_o_txt)) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  JointHandle* h = new JointHandle{};
  h->magic = kJointMagic;
  cudaGetDevice(&h->device);
  h->D = D;
  h->heads = heads;
  h->T = tp_degree;
  const size_t wq = size_t(3) * D * D * 2, wo = size_t(D) * D * 2;
  bool ok = cudaMalloc(&h->w_qkv_img, wq) == cudaSuccess && cudaMalloc(&h->w_qkv_txt, wq) == cudaSuccess &&
            cudaMalloc(&h->w_o_img, wo) == cudaSuccess && cudaMalloc(&h->w_o_txt, wo) == cudaSuccess;
  if (ok) {
    SliceJob sj[8];
    jobs_qkv_all(W_qkv_img, D, tp_degree, h->w_qkv_img, sj);
    jobs_qkv_all(W_qkv_txt, D, tp_degree, h->w_qkv_txt, sj + 3);
    sj[6] = job_rowwise_all(W_o_img, D, D, tp_degree, h->w_o_img);
    sj[7] = job_rowwise_all(W_o_txt, D, D, tp_degree, h->w_o_txt);
    ok = run_slice_jobs(sj, 8, s) == TP_OK;
  }
  if (!ok) {
    tp_destroy(h);
    return TP_ERR_CUDA;
  }
  *handle = h;
  return TP_OK;
}

tp_status tp_joint_attn_run(void* handle, const uint16_t* X_img, int64_t M_img, const uint16_t* X_txt, int64_t M_txt,
                            uint16_t* Y_img, uint16_t* Y_txt, void* ws, size_t ws_bytes, void* stream) {
  JointHandle* h = static_cast<JointHandle*>(handle);
  if (!h) return TP_ERR_BAD_HANDLE;
  if (h->magic != kJointMagic) return TP_ERR_BAD_HANDLE;
  if ((M_img > 0 && (!X_img || !Y_img)) || (M_txt > 0 && (!X_txt || !Y_txt))) return TP_ERR_NULL;
  tp_status st = check_joint_shape(M_img, M_txt, h->D, h->heads, h->T);
  if (st != TP_OK) return st;
  if (!al16(X_img) || !al16(X_txt) || !al16(Y_img) || !al16(Y_txt)) return TP_ERR_ALIGNMENT;
  if (M_img + M_txt == 0) return TP_OK;
  const JointLayout L = joint_layout(M_img + M_txt, h->D, false);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  uint8_t* w = static_cast<uint8_t*>(ws);
  return joint_attn_forward(di, X_img, M_img, X_txt, M_txt, h->D, h->heads, h->T, h->w_qkv_img, h->w_qkv_txt,
                            h->w_o_img, h->w_o_txt, reinterpret_cast<uint16_t*>(w + L.qkv),
                            reinterpret_cast<uint16_t*>(w + L.o), Y_img, Y_txt, as_stream(stream));
}

// ----------------------------------------------------------------------- context parallelism pieces
tp_status tp_sdpa_block_stats(const uint16_t* Q_qkv, int64_t Mq, const uint16_t* KV_qkv, int64_t Mk, int heads,
                              int tp_degree, uint16_t* O, float* lse, void* stream) {
  if (!Q_qkv || !KV_qkv || !O || !lse) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (Mq < 0 || Mk < 1 || heads < 1 || Mq >= kMaxDim || Mk >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (heads % tp_degree != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (!al16(Q_qkv) || !al16(KV_qkv) || !al16(O) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return run_sdpa_qkv(di, Q_qkv, Mq, KV_qkv, Mk, heads / tp_degree, tp_degree, O, true, lse, as_stream(stream));
}

tp_status tp_attn_merge(const uint16_t* O_parts, const float* lse_parts, int nparts, int64_t M, int heads,
                        int tp_degree, uint16_t* O, float* lse_out, void* stream) {
  if (!O_parts || !lse_parts || !O) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (nparts < 1 || nparts > 64 || M < 0 || heads < 1 || M >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (heads % tp_degree != 0) return TP_ERR_HEADS_INDIVISIBLE;
  if (!al16(O_parts) || !al16(O) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(lse_out) & 3u) != 0)
    return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  return launch_attn_merge(O_parts, lse_parts, nparts, M, heads / tp_degree, tp_degree, O, lse_out,
                           as_stream(stream)) == cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_unshard_rowwise_all(const uint16_t* src, int64_t rows, int64_t cols, int tp_degree, uint16_t* out,
                                 void* stream) {
  if (!src || !out) return TP_ERR_NULL;
  if (tp_degree < 1) return TP_ERR_BAD_DEGREE;
  if (rows < 1 || cols < 1 || rows >= kMaxDim || cols >= kMaxDim) return TP_ERR_BAD_SHAPE;
  if (cols % tp_degree != 0) return TP_ERR_INDIVISIBLE;
  const int64_t cs = cols / tp_degree;
  if (!al16(src) || !al16(out) || cs % 8 != 0) return TP_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  // block r of src ([rows x cs], contiguous) lands at columns [r*cs, (r+1)*cs) of out
  return launch_slice_copy(src, out, tp_degree, rows, cs, cs, rows * cs, cs, as_stream(stream), 1, 0, 0, cols) ==
                 cudaSuccess
             ? TP_OK
             : TP_ERR_CUDA;
}

// ----------------------------------------------------------------------- one rank's partial (multi-process TP)
size_t tp_mlp_rank_workspace_bytes(int64_t M, int64_t D, int64_t F, int tp_degree) {
  if (check_mlp_shape(M, D, F, tp_degree) != TP_OK) return 0;
  return mlp_rank_ws(M, F, tp_degree);
}

tp_status tp_mlp_rank_partial(const uint16_t* X, int64_t M, int64_t D, int64_t F, const uint16_t* W_up_r,
                              const uint16_t* b_up_r, const uint16_t* W_down_r, int tp_degree, float* part, void* ws,
                              size_t ws_bytes, void* stream) {
  if (!X || !W_up_r || !W_down_r || !part) return TP_ERR_NULL;
  tp_status st = check_mlp_shape(M, D, F, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(W_up_r) || !al16(W_down_r) || !al16(part) || (b_up_r && !al16(b_up_r)))
    return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  if ((st = check_ws(ws, ws_bytes, mlp_rank_ws(M, F, tp_degree))) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int64_t Fs = F / tp_degree;
  uint16_t* H = static_cast<uint16_t*>(ws);
  // this rank's colwise shard (one group) with bias + GELU, then its rowwise
  // partial (one K shard) left in fp32 for the cross-rank sum; no bias here
  if ((st = run_colwise(di, X, M, D, W_up_r, b_up_r, Fs, 1, 1, 0, H, s)) != TP_OK) return st;
  return run_rowwise(di, H, M, Fs, W_down_r, D, nullptr, 1, part, s, 0, true);
}

size_t tp_attn_rank_workspace_bytes(int64_t M, int64_t D, int heads, int tp_degree) {
  if (check_attn_shape(M, D, heads, tp_degree) != TP_OK) return 0;
  return attn_rank_layout(M, D, tp_degree).total;
}

tp_status tp_attn_rank_partial(const uint16_t* X, int64_t M, int64_t D, const uint16_t* W_qkv_r,
                               const uint16_t* W_o_r, int heads, int tp_degree, float* part, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!X || !W_qkv_r || !W_o_r || !part) return TP_ERR_NULL;
  tp_status st = check_attn_shape(M, D, heads, tp_degree);
  if (st != TP_OK) return st;
  if (!al16(X) || !al16(W_qkv_r) || !al16(W_o_r) || !al16(part)) return TP_ERR_ALIGNMENT;
  if (M == 0) return TP_OK;
  const AttnRankLayout L = attn_rank_layout(M, D, tp_degree);
  if ((st = check_ws(ws, ws_bytes, L.total)) != TP_OK) return st;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != TP_OK) return TP_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int64_t Ds = D / tp_degree;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* QKV = reinterpret_cast<uint16_t*>(w + L.qkv);
  uint16_t* O = reinterpret_cast<uint16_t*>(w + L.o);
  // this rank's heads only: QKV (fp16), SDPA over heads/T heads, rowwise partial in fp32
  if ((st = run_colwise(di, X, M, D, W_qkv_r, nullptr, 3 * Ds, 1, 0, 1, QKV, s)) != TP_OK) return st;
  if ((st = run_sdpa(di, QKV, M, heads / tp_degree, 1, O, s)) != TP_OK) return st;
  return run_rowwise(di, O, M, Ds, W_o_r, D, nullptr, 1, part, s, 0, true);
}

void tp_destroy(void* handle) {
  if (!handle) return;
  const uint64_t magic = *static_cast<uint64_t*>(handle);
  if (magic == kMlpMagic) {
    MlpHandle* h = static_cast<MlpHandle*>(handle);
    cudaDeviceSynchronize();
    cudaFree(h->w_up);
    cudaFree(h->b_up);
    cudaFree(h->w_down);
    cudaFree(h->b_down);
    h->magic = 0;
    delete h;
  } else if (magic == kAttnMagic) {
    AttnHandle* h = static_cast<AttnHandle*>(handle);
    cudaDeviceSynchronize();
    cudaFree(h->w_qkv);
    cudaFree(h->w_o);
    h->magic = 0;
    delete h;
  } else if (magic == kJointMagic) {
    JointHandle* h = static_cast<JointHandle*>(handle);
    cudaDeviceSynchronize();
    cudaFree(h->w_qkv_img);
    cudaFree(h->w_qkv_txt);
    cudaFree(h->w_o_img);
    cudaFree(h->w_o_txt);
    h->magic = 0;
    delete h;
  }
}

}  // extern "C"
