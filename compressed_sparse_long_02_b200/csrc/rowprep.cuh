// rowprep.cuh -- the per-row RMSNorm (unit gain) and partial RoPE shared by the
// compressor (entries, window rows), csa_norm_rope (queries) and the attention kernels'
// query preparation, so that every caller produces the same bits for the same row.
//
// Sources: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
// section 2.3 "Other details" (RMSNorm on query heads and KV entries right before core
// attention); dev.to "How DeepSeek-V4 Achieves ..." (partial rotary embedding on the last
// dimensions).
//
// A warp owns a row of C = 32 * CPT channels: lane l holds [l*CPT, (l+1)*CPT).  RoPE
// angles are reduced modulo 2 pi in double precision before a float sincos, so that
// positions up to 2^20 keep float accuracy.
#pragma once

#include <cuda_runtime.h>

namespace csa {
namespace rowprep {

constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

// theta^(-2i / rope_dims): the frequency of pair i
__device__ __forceinline__ double inv_freq(float theta, int i, int rope_dims) {
  return pow(static_cast<double>(theta), -2.0 * i / rope_dims);
}

// cos / sin of pos * inv_freq: the angle reduced modulo 2 pi in double, then a float sincos
__device__ __forceinline__ float2 rope_cs(double pos, double inv_freq) {
  const double ang = pos * inv_freq;
  const double k = rint(ang * kInvTwoPi);
  const float r = static_cast<float>(fma(-k, kTwoPi, ang));
  float s, c;
  sincosf(r, &s, &c);
  return make_float2(c, s);
}

// 1 / sqrt(mean of squares + eps) of a row held CPT channels per lane (all 32 lanes call it)
template <int CPT>
__device__ __forceinline__ float row_inv_rms(const float (&v)[CPT], int C, float eps) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < CPT; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  return 1.0f / sqrtf(ss / static_cast<float>(C) + eps);
}

// One round of the partial RoPE of the lane's channels [c0, c0 + CPT): pairs
// [base, base + 32) of the last rope_dims channels, lane l holding cs = (cos, sin) of pair
// base + l.  Pair (2i, 2i+1) turns by its angle; the lanes that own a pair fetch its angle
// by a shuffle.  All 32 lanes call.
template <int CPT>
__device__ __forceinline__ void rope_round(float (&v)[CPT], int c0, int C, int rope_dims, int base, float2 cs) {
  const int rope_base = C - rope_dims;
#pragma unroll
  for (int e = 0; e < CPT; e += 2) {
    const int c = c0 + e;
    const int pi = (c - rope_base) >> 1;  // this lane's pair at slot e (may be out of range)
    const int src = (pi - base) & 31;     // lane holding its angle in this round
    const float cx = __shfl_sync(0xffffffffu, cs.x, src);
    const float sx = __shfl_sync(0xffffffffu, cs.y, src);
    if (c >= rope_base && pi >= base && pi < base + 32) {
      const float r0 = fmaf(v[e], cx, -(v[e + 1] * sx));
      const float r1 = fmaf(v[e], sx, v[e + 1] * cx);
      v[e] = r0;
      v[e + 1] = r1;
    }
  }
}

// The partial RoPE at position pos: the angles are spread over the warp (lane l computes
// pairs l, l + 32, ...), so no lane computes more than ceil(pairs / 32) of them.
template <int CPT>
__device__ __forceinline__ void rope_lane(float (&v)[CPT], int c0, int C, int rope_dims, double pos,
                                          const double* inv_freq_tab) {
  const int npairs = rope_dims >> 1;
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < npairs; base += 32) {
    const int i = base + lane;
    const float2 cs = i < npairs ? rope_cs(pos, inv_freq_tab[i]) : make_float2(1.f, 0.f);
    rope_round<CPT>(v, c0, C, rope_dims, base, cs);
  }
}

}  // namespace rowprep
}  // namespace csa
