// noalloc.cu - tp_mlp_pair_sharded_noalloc: the MLP pair with no device
// allocation anywhere on its path.
//
// For callers that must not allocate device memory (see include/tp.h: memory
// owned by another allocator, or no tolerance for the synchronisation that
// cudaMalloc/cudaFree may cause).  The FFN hidden activations, which
// tp_mlp_run keeps in a caller workspace, live here in a fixed file-scope
// device array instead; tokens are processed in row chunks whose activations
// fit in it.  The kernels are the same colwise and rowwise tcgen05 GEMMs as
// every other path, so each token's result is the same arithmetic in the same
// order as tp_mlp_pair.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/tp.h"
#include "internal.h"

namespace tp {
namespace {

constexpr size_t kScratchBytes = size_t(TP_NOALLOC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;
constexpr int64_t kChunkAlign = 128;  // GEMM tile height

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address comes from cudaGetSymbolAddress.
// This file holds no kernel, so under CUDA's lazy module loading (the default)
// the driver creates the array on a device when its address is first looked
// up there, i.e. inside the first call on that device; with eager loading it
// exists as soon as the library's modules are loaded.
static __device__ __align__(256) uint16_t g_noalloc_scratch[kScratchBytes / sizeof(uint16_t)];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up once per device.
tp_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return TP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" tp_status tp_mlp_pair_sharded_noalloc(const uint16_t* X, int64_t M, int64_t D, int64_t F,
                                                 const uint16_t* W_up_shards, const uint16_t* b_up_shards,
                                                 const uint16_t* W_down_shards, const uint16_t* b_down,
                                                 int tp_degree, uint16_t* Y, void* stream) {
  if (!X || !W_up_shards || !W_down_shards || !Y) return TP_ERR_NULL;
  // The same shape rules as every other MLP entry point (one shared check).
  const int shape = mlp_shape_status(M, D, F, tp_degree);
  if (shape != TP_OK) return tp_status(shape);
  const int64_t Fs = F / tp_degree;
  if (!aligned16(X) || !aligned16(W_up_shards) || !aligned16(W_down_shards) || !aligned16(Y) ||
      (b_up_shards && !aligned16(b_up_shards)) || (b_down && !aligned16(b_down)))
    return TP_ERR_ALIGNMENT;
  // One token's activations across all shards take 2*F bytes; a chunk must hold
  // at least one 128-row tile of them.
  const int64_t row_bytes = 2 * F;
  if (row_bytes * kChunkAlign > int64_t(kScratchBytes)) return TP_ERR_SCRATCH_LIMIT;
  if (M == 0) return TP_OK;
  const int64_t chunk = (int64_t(kScratchBytes) / row_bytes) / kChunkAlign * kChunkAlign;

  int num_sms = 0;
  int* err = nullptr;
  if (current_device_context(&num_sms, &err) != TP_OK) return TP_ERR_CUDA;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != TP_OK) return TP_ERR_CUDA;
  uint16_t* H = static_cast<uint16_t*>(scratch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const GemmOperand wup{W_up_shards, uint64_t(D), uint64_t(Fs), uint64_t(tp_degree)};
  const GemmOperand wdown{W_down_shards, uint64_t(Fs), uint64_t(D), uint64_t(tp_degree)};

  for (int64_t m0 = 0; m0 < M; m0 += chunk) {
    const int64_t mc = (M - m0) < chunk ? (M - m0) : chunk;
    // colwise: H[r][0:mc] = GELU(X[m0:m0+mc] . W_up,r^T + b_up,r) for every shard r
    const GemmOperand xop{X + m0 * D, uint64_t(D), uint64_t(mc), 1};
    const GemmOperand hop{H, uint64_t(Fs), uint64_t(mc), uint64_t(tp_degree)};
    GemmArgs c{};
    c.M = int(mc);
    c.N = int(Fs);
    c.k_blocks = int((D + 63) / 64);
    c.kshards = 1;
    c.groups = tp_degree;
    c.a_follows_shard = 0;
    c.out = H;
    c.out_gstride = mc * Fs;
    c.ldo = Fs;
    c.bias = b_up_shards;
    c.bias_gstride = Fs;
    c.gelu = 1;
    c.out_f16 = 0;
    c.err = err;
    if (launch_gemm(xop, wup, c, num_sms, s) != cudaSuccess) return TP_ERR_CUDA;
    // rowwise: Y[m0:m0+mc] = sum_r H[r][0:mc] . W_down,r^T + b_down
    GemmArgs r{};
    r.M = int(mc);
    r.N = int(D);
    r.k_blocks = int((Fs + 63) / 64);
    r.kshards = tp_degree;
    r.groups = 1;
    r.a_follows_shard = 1;
    r.out = Y + m0 * D;
    r.out_gstride = 0;
    r.ldo = D;
    r.bias = b_down;
    r.bias_gstride = 0;
    r.gelu = 0;
    r.out_f16 = 0;
    r.err = err;
    if (launch_gemm(hop, wdown, r, num_sms, s) != cudaSuccess) return TP_ERR_CUDA;
  }
  return TP_OK;
}
