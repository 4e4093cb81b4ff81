// selftest.cu -- csa_selftest_bounded_wait: runs the bounded mbarrier waits that every
// pipeline of this library uses against barriers that never complete, so the host can
// check the failure-detection path without faulting or hanging the GPU.
//
// One CTA of two warps.  Warp 0 waits on barrier A, which nothing ever arrives on; after
// the wait limit it records CSA_DEVERR_TIMEOUT in the device error word, raises the CTA's
// abort flag and returns false.  Warp 1 waits on barrier B, which nothing arrives on
// either; it is released by the abort flag (the way every other role of a pipeline is
// released when one role gives up) and returns false without a second timeout of its own.
// Warp 1 starts waiting a quarter of the limit later than warp 0.  Each warp then writes
// its result and the SM cycles it waited; the kernel exits normally and the context stays
// usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "csa.h"
#include "internal.h"
#include "ptx.cuh"

namespace csa {
namespace {

__global__ void bounded_wait_kernel(int sleeping, int32_t* err, long long* out) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 1) {
    // start a quarter of the limit after warp 0, so that warp 0 reaches the limit first and
    // warp 1 is released by the abort flag before its own limit
    const long long s0 = clock64();
    while (clock64() - s0 < kWaitLimitCycles / 4) __nanosleep(100000);
  }
  const long long t0 = clock64();
  const bool ok = sleeping ? warp_wait_sleep(&bars[warp], 0, err, abort_flag)
                           : warp_wait(&bars[warp], 0, err, abort_flag);
  const long long dt = clock64() - t0;
  if (lane == 0) {
    out[2 * warp] = ok ? 1 : 0;
    out[2 * warp + 1] = dt;
  }
}

}  // namespace
}  // namespace csa

extern "C" csa_status csa_selftest_bounded_wait(int sleeping, long long* out, cudaStream_t stream) {
  using namespace csa;
  if (out == nullptr || (sleeping != 0 && sleeping != 1)) return CSA_ERR_INVALID_ARG;
  int32_t* err = device_error_word();
  if (err == nullptr) return CSA_ERR_CUDA;
  bounded_wait_kernel<<<1, 64, 0, stream>>>(sleeping, err, out);
  return status_from_cuda(cudaGetLastError());
}
