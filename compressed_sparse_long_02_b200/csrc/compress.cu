// compress.cu -- softmax-weighted KV pooling (CSA m=4 with the previous group
// overlapped, HCA m'=128), RMSNorm, partial RoPE and the fused MXFP4 encoding of
// indexer keys; plus the row-wise RMSNorm + RoPE used for queries and raw window rows.
//
// Sources: "DeepSeek-V4: Million-Token Context" (CSA stage: m=4 tokens pooled by a
// learned softmax weighting; HCA stage: m'=128), "Follow the white rabbit: DeepSeek
// V4's architecture in 3D" (CSA entries also draw on the previous group of four; HCA
// weights differ across parts of the representation), "DeepSeek-V4: Towards Highly
// Efficient Million-Token Context Intelligence" section 2.3 (RMSNorm on queries and
// entries before core attention; partial RoPE).
//
// Design: both kernels are HBM-bound.  One thread owns a pair of adjacent channels
// (so a RoPE pair never crosses threads and each load is 4 or 8 bytes, coalesced
// across the CTA); each token row is read once per entry that pools it.  Angles
// are reduced in double precision before a float sincos so that positions up to
// 2^20 keep float accuracy.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"

namespace csa {
namespace {

constexpr double kTwoPi = 6.283185307179586476925286766559;

__device__ __forceinline__ float2 rope_cs(double pos, double inv_freq) {
  double ang = pos * inv_freq;
  double k = rint(ang / kTwoPi);
  float r = static_cast<float>(fma(-k, kTwoPi, ang));
  float s, c;
  sincosf(r, &s, &c);
  return make_float2(c, s);
}

template <bool kBf16>
__device__ __forceinline__ float2 load_pair(const void* base, size_t off) {
  if constexpr (kBf16) {
    uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(base) + off));
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
  } else {
    return __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(base) + off));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// one CTA = `epc` consecutive entries of one sequence; thread = channel pair.  In
// streaming mode (a.pos set) a CTA serves one sequence and writes at most the one entry
// its newest token completes, from the sequence's last S raw rows.
template <bool kBf16>
__global__ void pool_kernel(PoolArgs a, int epc) {
  griddep_enter();
  __shared__ float red[32];
  const int b = blockIdx.y;
  const int C = a.C;
  const int c0 = 2 * threadIdx.x;
  const int S = a.overlap ? 2 * a.m : a.m;
  const bool stream = a.pos != nullptr;
  int E = a.T / a.m, j_stream = 0, tok_ring = 0;
  if (stream) {  // uniform over the CTA
    const int pos = a.pos[b];
    if (pos < 0 || (pos + 1) % a.m != 0) return;  // no group completes at this token
    j_stream = (pos + 1) / a.m - 1;
    if (j_stream >= a.E_max) {
      if (threadIdx.x == 0) atomicExch(a.err, CSA_DEVERR_INDEX);
      return;
    }
    tok_ring = pos - S + 1;  // token of ring row 0
    E = j_stream + 1;
  }
  const int rope_base = C - a.rope_dims;
  const bool rot = a.rope_dims > 0 && c0 >= rope_base;
  const double inv_freq = rot ? pow(static_cast<double>(a.theta), -2.0 * ((c0 - rope_base) / 2) / a.rope_dims) : 0.0;

  for (int jj = 0; jj < epc; ++jj) {
    const int j = stream ? j_stream : blockIdx.x * epc + jj;
    if (j >= E) break;  // uniform over the CTA
    const int first = a.overlap ? a.m * (j - 1) : a.m * j;
    float mx0 = -INFINITY, mx1 = -INFINITY, den0 = 0.f, den1 = 0.f, num0 = 0.f, num1 = 0.f;
#pragma unroll 4
    for (int s = 0; s < S; ++s) {
      const int tok = first + s;
      if (tok < 0) continue;  // previous group of entry 0 does not exist: excluded
      const size_t row = stream ? static_cast<size_t>(b) * S + (tok - tok_ring) : static_cast<size_t>(b) * a.T + tok;
      const size_t off = row * C + c0;
      const float2 x = load_pair<kBf16>(a.kv, off);
      const float2 z = load_pair<kBf16>(a.logits, off);
      const float2 bs = __ldg(reinterpret_cast<const float2*>(a.bias + static_cast<size_t>(s) * C + c0));
      const float a0 = z.x + bs.x, a1 = z.y + bs.y;
      if (a0 > mx0) {
        const float r = expf(mx0 - a0);
        den0 = den0 * r + 1.f;
        num0 = num0 * r + x.x;
        mx0 = a0;
      } else {
        const float e = expf(a0 - mx0);
        den0 += e;
        num0 = fmaf(e, x.x, num0);
      }
      if (a1 > mx1) {
        const float r = expf(mx1 - a1);
        den1 = den1 * r + 1.f;
        num1 = num1 * r + x.y;
        mx1 = a1;
      } else {
        const float e = expf(a1 - mx1);
        den1 += e;
        num1 = fmaf(e, x.y, num1);
      }
    }
    float e0 = num0 / den0, e1 = num1 / den1;
    const size_t eoff = (static_cast<size_t>(b) * a.E_max + j) * C + c0;

    if (a.fp4 != nullptr) {  // indexer key cache: pooled values before norm / RoPE
      uint8_t byte, sbyte;
      mxfp4_encode_pair(e0, e1, byte, sbyte);
      a.fp4[eoff / 2] = byte;
      if ((threadIdx.x & 15) == 0) a.fp4_scale[eoff / 32] = sbyte;
    }
    if (a.entries != nullptr) {
      if (a.norm) {
        const float ss = block_sum(e0 * e0 + e1 * e1, red);
        const float inv = 1.0f / sqrtf(ss / C + a.eps);
        e0 *= inv;
        e1 *= inv;
      }
      if (rot) {
        const float2 cs = rope_cs(static_cast<double>(a.m) * (j + 1) - 1.0, inv_freq);
        const float r0 = e0 * cs.x - e1 * cs.y;
        const float r1 = e0 * cs.y + e1 * cs.x;
        e0 = r0;
        e1 = r1;
      }
      reinterpret_cast<uint32_t*>(a.entries)[eoff / 2] = pack_bf16x2(e0, e1);
    }
    if (stream) break;
  }
}

// one CTA = one row (all heads); one warp per head vector, EPL consecutive channels per lane
template <bool kBf16, int EPL>
__global__ void norm_rope_kernel(NormRopeArgs a) {
  griddep_enter();
  extern __shared__ float2 cs[];  // [rope_dims/2] (cos, sin) for this row's position
  const int64_t row = blockIdx.x;
  const int C = a.C;
  const int64_t pos = a.pos ? static_cast<int64_t>(a.pos[row]) : row % a.pos_mod;
  const int npairs = a.rope_dims / 2;
  for (int i = threadIdx.x; i < npairs; i += blockDim.x)
    cs[i] = rope_cs(static_cast<double>(pos), pow(static_cast<double>(a.theta), -2.0 * i / a.rope_dims));
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int rope_base = C - a.rope_dims;
  for (int h = warp; h < a.heads; h += nw) {
    const size_t base = (static_cast<size_t>(row) * a.heads + h) * C + lane * EPL;
    float v[EPL];
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 p = load_pair<kBf16>(a.x, base + e);
      v[e] = p.x;
      v[e + 1] = p.y;
    }
    if (a.norm) {
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.0f / sqrtf(ss / C + a.eps);
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] *= inv;
    }
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const int c = lane * EPL + e;
      if (a.rope_dims > 0 && c >= rope_base) {
        const float2 t = cs[(c - rope_base) / 2];
        const float r0 = v[e] * t.x - v[e + 1] * t.y;
        const float r1 = v[e] * t.y + v[e + 1] * t.x;
        v[e] = r0;
        v[e + 1] = r1;
      }
    }
    uint32_t* o = reinterpret_cast<uint32_t*>(a.out + base);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) o[e / 2] = pack_bf16x2(v[e], v[e + 1]);
  }
}

template <bool kBf16>
cudaError_t launch_norm_rope_t(const NormRopeArgs& a, cudaStream_t s) {
  const int warps = a.heads < 8 ? a.heads : 8;
  const dim3 grid(static_cast<unsigned>(a.rows)), block(32 * warps);
  const size_t smem = sizeof(float2) * (a.rope_dims / 2 > 0 ? a.rope_dims / 2 : 1);
  cudaError_t e = cudaSuccess;
  switch (a.C / 32) {
    case 2: e = launch_pdl(norm_rope_kernel<kBf16, 2>, grid, block, smem, s, a); break;
    case 4: e = launch_pdl(norm_rope_kernel<kBf16, 4>, grid, block, smem, s, a); break;
    case 8: e = launch_pdl(norm_rope_kernel<kBf16, 8>, grid, block, smem, s, a); break;
    case 16: e = launch_pdl(norm_rope_kernel<kBf16, 16>, grid, block, smem, s, a); break;
    case 32: e = launch_pdl(norm_rope_kernel<kBf16, 32>, grid, block, smem, s, a); break;
    default: return cudaErrorInvalidValue;
  }
  return e;
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  return a.in_bf16 ? launch_norm_rope_t<true>(a, s) : launch_norm_rope_t<false>(a, s);
}

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s) {
  if (a.entries == nullptr && a.fp4 == nullptr) return cudaSuccess;
  if (a.pos != nullptr) {  // streaming: one CTA per sequence
    const dim3 grid(1, a.B), block(a.C / 2);
    return a.in_bf16 ? launch_pdl(pool_kernel<true>, grid, block, 0, s, a, 1)
                     : launch_pdl(pool_kernel<false>, grid, block, 0, s, a, 1);
  }
  const int E = a.T / a.m;
  if (E == 0) return cudaSuccess;
  const int epc = a.m >= 32 ? 1 : (a.m >= 8 ? 4 : 16);
  const dim3 grid((E + epc - 1) / epc, a.B), block(a.C / 2);
  return a.in_bf16 ? launch_pdl(pool_kernel<true>, grid, block, 0, s, a, epc)
                   : launch_pdl(pool_kernel<false>, grid, block, 0, s, a, epc);
}

}  // namespace csa
