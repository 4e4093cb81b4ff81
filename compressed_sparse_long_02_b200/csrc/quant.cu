// quant.cu -- MXFP4 encoding of an activation matrix (indexer queries and keys).
//
// HBM-bound.  A thread encodes units of 8 consecutive elements (one 16-byte bf16 load
// or two float32 loads) into 4 packed bytes; four consecutive lanes hold one 32-element
// block and agree on its scale through two shuffles, and the block's first lane writes
// the scale byte.  A warp covers 256 consecutive elements per unit, so every load and
// store instruction of the warp is contiguous; each thread keeps kUnits units in flight.
// The E2M1 rounding is the hardware conversion of the exactly scaled values (mxfp4.cuh).
#include <cuda_runtime.h>

#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"

namespace csa {
namespace {

constexpr int kQuantThreads = 256;

template <bool kBf16>
__device__ __forceinline__ void load8(const void* x, int64_t unit, float (&v)[8]) {
  if constexpr (kBf16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x) + unit);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * unit);
    const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * unit + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// n_units = elements / 8 (a multiple of 4: whole 32-element blocks).  The rounds of a warp
// are uniform over its lanes, so the shuffles of a round always have all 32 lanes.
template <bool kBf16, int kUnits>  // kUnits: units of 8 elements in flight per thread
__global__ void __launch_bounds__(kQuantThreads) quantize_mxfp4_kernel(const void* __restrict__ x, int64_t n_units,
                                                                       uint8_t* __restrict__ packed,
                                                                       uint8_t* __restrict__ scales) {
  griddep_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  // round r of warp w covers units [(r * n_warps + w) * 32 * kUnits, +32 * kUnits)
  for (int64_t base = warp_g * 32 * kUnits; base < n_units; base += n_warps * 32 * kUnits) {
    float v[kUnits][8];
#pragma unroll
    for (int u = 0; u < kUnits; ++u) {  // every load of the round in flight first
      const int64_t unit = base + u * 32 + lane;
      if (unit < n_units) {
        load8<kBf16>(x, unit, v[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnits; ++u) {
      const int64_t unit = base + u * 32 + lane;
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[u][i]));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      const int E = mx_block_exponent(am);
      const uint32_t word = e2m1x8_rn(v[u], mx_pow2_neg(E));
      if (unit < n_units) {
        reinterpret_cast<uint32_t*>(packed)[unit] = word;
        if ((lane & 3) == 0) scales[unit >> 2] = static_cast<uint8_t>(E + 127);
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_mxfp4(const void* x, int in_bf16, int64_t rows, int cols, uint8_t* packed,
                                  uint8_t* scales, cudaStream_t s) {
  const int64_t n_units = rows * (cols / 8);
  if (n_units == 0) return cudaSuccess;
  // large inputs: four units in flight per thread; small ones (a decode step's queries):
  // one, so that the work spreads over more CTAs
  const bool small = n_units < static_cast<int64_t>(num_sms()) * kQuantThreads * 4;
  const int64_t per_cta = static_cast<int64_t>(kQuantThreads) * (small ? 1 : 4);
  int64_t blocks = (n_units + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks)), block(kQuantThreads);
  if (small)
    return in_bf16 ? launch_pdl(quantize_mxfp4_kernel<true, 1>, grid, block, 0, s, x, n_units, packed, scales)
                   : launch_pdl(quantize_mxfp4_kernel<false, 1>, grid, block, 0, s, x, n_units, packed, scales);
  return in_bf16 ? launch_pdl(quantize_mxfp4_kernel<true, 4>, grid, block, 0, s, x, n_units, packed, scales)
                 : launch_pdl(quantize_mxfp4_kernel<false, 4>, grid, block, 0, s, x, n_units, packed, scales);
}

}  // namespace csa
