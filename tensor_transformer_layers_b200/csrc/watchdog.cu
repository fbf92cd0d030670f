// watchdog.cu - exercises the kernels' bounded-wait path on the GPU.
//
// Every mbarrier wait in this library gives up after a time limit, records
// kErrTimeout in the device error word and lets the kernel return, so that a
// lost arrival shows up as TP_ERR_DEVICE_TIMEOUT from tp_check_device_error()
// instead of a hung GPU.  This kernel waits, through the same bounded wait, on
// an mbarrier that nothing ever arrives on: the wait must run out, the error
// word must be set and the kernel must finish.  No fault, trap or unbounded
// loop is involved.
#include "internal.h"
#include "ptx.cuh"

namespace tp {
namespace {

__global__ void watchdog_probe_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Phase 0 never completes: nothing arrives on `bar`.
    if (!mbar_wait_for(&bar, 0, &abort_flag, limit_ns)) report_timeout(err, &abort_flag);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_watchdog_probe(int* err, uint64_t limit_ns, cudaStream_t s) {
  watchdog_probe_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  count_launch();
  return note_cuda_error("watchdog probe: launch", cudaGetLastError());
}

}  // namespace tp
