// peak.cu -- dense tcgen05 throughput probe: the measured denominator for the
// contractions of this library whose datatype has no library-measured peak (the
// block-scaled FP4 indexer), with the same probe in bf16 beside it to compare with a
// library GEMM's measured bf16 rate.
//
// One CTA per SM.  Operand tiles are written once into shared memory (A: 128 rows x
// 128 bytes, B: N rows x 128 bytes, K-major, SWIZZLE_128B); one thread then issues
// `iters` rounds of four MMAs over the tiles (M = 128, N as given, K = 4 x 64 FP4 or
// 4 x 16 bf16 elements) into one TMEM accumulator, commits and waits.  No global memory
// is read in the loop: the rate is the tensor pipe's alone.  Operand values do not
// matter for the rate (the tiles hold a fixed byte pattern, the scale factors 2^-127).
#include <cuda_runtime.h>

#include <cstdint>

#include "csa.h"
#include "internal.h"
#include "ptx.cuh"

namespace csa {
namespace {

constexpr int kPeakThreads = 128;
constexpr uint32_t kPeakTmemCols = 512;  // accumulator [0, 256), scale factors at 256 and 288
constexpr size_t kPeakSmem = 1024 + 16384 + 32768 + 1024 + 64;

__global__ void __launch_bounds__(kPeakThreads, 1) mma_peak_kernel(int mxf4, int N, int iters, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                  // 128 x 128 B
  uint8_t* sB = sA + 16384;            // N x 128 B, N <= 256
  uint8_t* sSF = sB + 32768;           // 1 KB of zero scale bytes
  uint64_t* done = reinterpret_cast<uint64_t*>(sSF + 1024);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_word = reinterpret_cast<int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += kPeakThreads)
    reinterpret_cast<uint4*>(sA)[i] = make_uint4(0x22222222u, 0x11111111u, 0x33333333u, 0x11111111u);
  for (int i = threadIdx.x; i < 1024 / 16; i += kPeakThreads) reinterpret_cast<uint4*>(sSF)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPeakTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const uint32_t sfa = tmem + 256, sfb = tmem + 288;
    if (mxf4) {
      tc_cp_32x128b_warpx4(sfa, smem_desc(smem_u32(sSF), 0, 128, kSwizzleNone));
      for (int c = 0; c < 8; c += 4) tc_cp_32x128b_warpx4(sfb + c, smem_desc(smem_u32(sSF), 0, 128, kSwizzleNone));
    }
    const uint32_t idesc = mxf4 ? idesc_mxf4(128, N, 0, 0) : idesc_bf16(128, N, false, false);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = smem_desc(a0 + 32 * kk, 16, 1024, kSwizzle128B);
        const uint64_t db = smem_desc(b0 + 32 * kk, 16, 1024, kSwizzle128B);
        const uint32_t acc = (it | kk) ? 1u : 0u;
        if (mxf4)
          mma_mxf4(tmem, da, db, idesc, acc, sfa, sfb);
        else
          mma_bf16(tmem, da, db, idesc, acc);
      }
    }
    tc_commit(done);
    mbar_wait(done, 0, err, abort_word);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPeakTmemCols);
  }
}

int g_peak_smem[64];

}  // namespace
}  // namespace csa

extern "C" csa_status csa_mma_peak_probe(int mxf4, int N, int iters, int ctas, double* flops_out,
                                         cudaStream_t stream) {
  using namespace csa;
  if ((mxf4 != 0 && mxf4 != 1) || N < 16 || N > 256 || N % 16 != 0 || iters < 1 || ctas < 1)
    return CSA_ERR_INVALID_ARG;
  int32_t* err = device_error_word();
  if (err == nullptr) return CSA_ERR_CUDA;
  cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(mma_peak_kernel), kPeakSmem, g_peak_smem);
  if (e != cudaSuccess) return status_from_cuda(e);
  mma_peak_kernel<<<ctas, kPeakThreads, kPeakSmem, stream>>>(mxf4, N, iters, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return status_from_cuda(e);
  const double k_per_round = mxf4 ? 4.0 * 64.0 : 4.0 * 16.0;
  if (flops_out) *flops_out = 2.0 * 128.0 * N * k_per_round * iters * ctas;
  return CSA_OK;
}
