// quant.cu -- MXFP4 encoding of an activation matrix (indexer queries and keys).
// HBM-bound: each thread reads two elements (one output byte), 16 lanes form one
// 32-element block and agree on its scale through shuffles.
#include <cuda_runtime.h>

#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"

namespace csa {
namespace {

template <bool kBf16>
__global__ void quantize_mxfp4_kernel(const void* __restrict__ x, int64_t n_pairs, uint8_t* __restrict__ packed,
                                      uint8_t* __restrict__ scales) {
  griddep_enter();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // the loop trip count is uniform across each warp because n_pairs % 16 == 0 and the
  // grid covers whole warps
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g - threadIdx.x % 32 < n_pairs;
       g += stride) {
    const bool live = g < n_pairs;
    float x0 = 0.f, x1 = 0.f;
    if (live) {
      if constexpr (kBf16) {
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(x) + g);
        x0 = __uint_as_float(u << 16);
        x1 = __uint_as_float(u & 0xFFFF0000u);
      } else {
        const float2 p = __ldg(reinterpret_cast<const float2*>(x) + g);
        x0 = p.x;
        x1 = p.y;
      }
    }
    uint8_t byte, sbyte;
    mxfp4_encode_pair(x0, x1, byte, sbyte);
    if (live) {
      packed[g] = byte;
      if ((g & 15) == 0) scales[g >> 4] = sbyte;
    }
  }
}

}  // namespace

cudaError_t launch_quantize_mxfp4(const void* x, int in_bf16, int64_t rows, int cols, uint8_t* packed,
                                  uint8_t* scales, cudaStream_t s) {
  const int64_t n_pairs = rows * (cols / 2);
  if (n_pairs == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (n_pairs + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (in_bf16)
    return launch_pdl(quantize_mxfp4_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s, x, n_pairs, packed, scales);
  else
    return launch_pdl(quantize_mxfp4_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s, x, n_pairs, packed, scales);
}

}  // namespace csa
