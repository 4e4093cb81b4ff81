// compress.cu -- softmax-weighted KV pooling (CSA m=4 with the previous group
// overlapped, HCA m'=128), RMSNorm, partial RoPE and the fused MXFP4 encoding of
// indexer keys, with the raw-token window rows written in the same pass; plus the
// row-wise RMSNorm + RoPE used for queries (and for a decode token's window row).
//
// Sources: "DeepSeek-V4: Million-Token Context" (CSA stage: m=4 tokens pooled by a
// learned softmax weighting; HCA stage: m'=128), "Follow the white rabbit: DeepSeek
// V4's architecture in 3D" (CSA entries also draw on the previous group of four; HCA
// weights differ across parts of the representation; the most recent 128 raw tokens are
// kept for the sliding window), "DeepSeek-V4: Towards Highly Efficient Million-Token
// Context Intelligence" section 2.3 (RMSNorm on queries and entries before core
// attention; partial RoPE).
//
// Both kernels are HBM-bound.  A warp owns whole rows: lane l holds the CPT = C/32
// consecutive channels [l*CPT, (l+1)*CPT), loaded with the widest vector loads the row
// allows (16 bytes for C = 512 bf16), so a row's RMSNorm is a warp reduction and a RoPE
// pair never crosses lanes.  pool_kernel gives each entry one warp (CSA: its 8 slots)
// or eight warps (HCA: 16 of its 128 slots each, merged through shared memory), keeps
// the per-channel softmax state in registers (updated a chunk of slots at a time: one
// rescale, then one exponential per slot), and writes the window row of every token
// of the entry's own group while that row is in registers, so kv is read from HBM once
// (the overlapped previous group's rows are read again from L2).
//
// The window rows written here and the rows csa_norm_rope writes (a decode token's
// window row) go through the same per-row helpers in the same order, so the two are
// bitwise equal.  RoPE angles are reduced in double precision before a float sincos so
// that positions up to 2^20 keep float accuracy.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"
#include "rowprep.cuh"

namespace csa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPoolThreads = 256;  // 8 warps
// slots loaded together and pooled as one chunk: 4, fewer when a lane's row slice is
// large, so that the rows in flight and the softmax state fit the registers of two CTAs
// per SM (C = 512 bf16, 8 words a lane: 2 -- measured 13 % faster than 4 for HCA 64K,
// equal for CSA 8K)
template <int kWords>
constexpr int pool_chunk() {
  return kWords >= 32 ? 1 : (kWords >= 8 ? 2 : 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// The CPT channels a lane holds of one row, as raw words (bf16 pairs or float32).
template <bool kBf16, int CPT>
struct RowBits {
  static constexpr int kBytes = CPT * (kBf16 ? 2 : 4);
  static constexpr int kWords = kBytes / 4;
  static_assert(kWords >= 1, "at least one word per lane");
  uint32_t w[kWords];
  // row: start of a row of C = 32 * CPT elements
  __device__ __forceinline__ void load(const void* row, int lane) {
    const uint8_t* p = static_cast<const uint8_t*>(row) + lane * kBytes;
    if constexpr (kBytes % 16 == 0) {
#pragma unroll
      for (int i = 0; i < kBytes / 16; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
    } else if constexpr (kBytes == 8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = v.x;
      w[1] = v.y;
    } else {
      w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = 0u;
  }
  __device__ __forceinline__ float get(int i) const {
    if constexpr (kBf16) {
      const uint32_t u = w[i >> 1];
      return (i & 1) ? __uint_as_float(u & 0xFFFF0000u) : __uint_as_float(u << 16);
    } else {
      return __uint_as_float(w[i]);
    }
  }
};

using rowprep::rope_lane;
using rowprep::row_inv_rms;

// RMSNorm (optional) + RoPE of one row, stored as bf16 at out_row + lane's channels
template <int CPT>
__device__ __forceinline__ void norm_rope_store(float (&v)[CPT], int lane, int C, int norm, float eps,
                                                int rope_dims, double pos, const double* inv_freq,
                                                uint16_t* out_row) {
  if (norm) {
    const float inv = row_inv_rms<CPT>(v, C, eps);
#pragma unroll
    for (int e = 0; e < CPT; ++e) v[e] *= inv;
  }
  rope_lane<CPT>(v, lane * CPT, C, rope_dims, pos, inv_freq);
  uint32_t w[CPT / 2];
#pragma unroll
  for (int e = 0; e < CPT; e += 2) w[e / 2] = pack_bf16x2(v[e], v[e + 1]);
  uint16_t* dst = out_row + lane * CPT;
  if constexpr (CPT >= 8) {
#pragma unroll
    for (int i = 0; i < CPT / 8; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  } else if constexpr (CPT == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = w[0];
  }
}

// MXFP4 encoding of the lane's CPT pooled values; a 32-element block spans 32 / CPT lanes
// (one lane when CPT = 32), whose amax is combined by shuffles.  Bytes: element 2i in the
// low nibble; one scale byte per block, written by the block's first lane.
template <int CPT>
__device__ __forceinline__ void fp4_store(const float (&v)[CPT], int lane, uint8_t* packed_row, uint8_t* scale_row) {
  float am = 0.f;
#pragma unroll
  for (int e = 0; e < CPT; ++e) am = fmaxf(am, fabsf(v[e]));
  constexpr int kLanesPerBlock = CPT >= 32 ? 1 : 32 / CPT;
#pragma unroll
  for (int o = 1; o < kLanesPerBlock; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int E = mx_block_exponent(am);
  const float inv_T = mx_pow2_neg(E);
  uint8_t bytes[CPT / 2];
#pragma unroll
  for (int e = 0; e < CPT; e += 2) bytes[e / 2] = static_cast<uint8_t>(e2m1x2_rn(v[e] * inv_T, v[e + 1] * inv_T));
  uint8_t* dst = packed_row + lane * (CPT / 2);
  if constexpr (CPT == 32) {
    uint4 q;
    memcpy(&q, bytes, 16);
    *reinterpret_cast<uint4*>(dst) = q;
  } else if constexpr (CPT == 16) {
    uint2 q;
    memcpy(&q, bytes, 8);
    *reinterpret_cast<uint2*>(dst) = q;
  } else if constexpr (CPT == 8) {
    uint32_t q;
    memcpy(&q, bytes, 4);
    *reinterpret_cast<uint32_t*>(dst) = q;
  } else if constexpr (CPT == 4) {
    uint16_t q;
    memcpy(&q, bytes, 2);
    *reinterpret_cast<uint16_t*>(dst) = q;
  } else {
    *dst = bytes[0];
  }
  if ((lane * CPT) % 32 == 0) scale_row[lane * CPT / 32] = static_cast<uint8_t>(E + 127);
}

// 2^x by the hardware approximation (relative error ~2^-22); the pooled value is a ratio
// of two sums of these, rounded to bf16 afterwards.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A chunk of U slots of one channel: logits a[u] (log2 units, -inf for a slot that does
// not exist, at least one does) with chunk maximum cm, values x[u].get(e).  The running
// state is rescaled once to the new maximum, then each slot adds 2^(a - max).
template <int U, typename Rows>
__device__ __forceinline__ void softmax_chunk(const float (&av)[U], const Rows (&x)[U], int e, float cm, float& mx,
                                              float& den, float& num) {
  const float nm = fmaxf(mx, cm);  // finite: the chunk has a slot
  const float r = fast_exp2(mx - nm);  // mx = -inf: 0
  float d = den * r, n = num * r;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const float pr = fast_exp2(av[u] - nm);  // a slot that does not exist: 2^-inf = 0
    d += pr;
    n = fmaf(pr, x[u].get(e), n);
  }
  den = d;
  num = n;
  mx = nm;
}

size_t pool_smem_bytes(int C, int rope_dims, int split) {
  return static_cast<size_t>(rope_dims / 2) * sizeof(double) + (split > 1 ? static_cast<size_t>(split) * 3 * C * 4 : 0);
}

// Grid (ceil(groups / entries per CTA), B); 256 threads.  kSplit warps pool one entry,
// each over a contiguous part of the entry's slots (merged through shared memory when
// kSplit > 1).  Group j of a sequence: tokens [m j, m j + m); groups past the last
// complete one (j >= floor(T/m)) exist only to write window rows of a trailing partial
// group.  Streaming mode (a.pos set): one CTA per sequence, the entry its newest token
// completes, rows from the sequence's ring of its last S raw tokens; no window rows.
template <bool kBf16, int CPT, int kSplit>
__global__ void __launch_bounds__(kPoolThreads, 2) pool_kernel(PoolArgs a) {
  extern __shared__ __align__(16) uint8_t pool_smem[];
  double* inv_freq = reinterpret_cast<double*>(pool_smem);
  float* part = reinterpret_cast<float*>(pool_smem + (a.rope_dims / 2) * sizeof(double));  // [kSplit][3][C]
  for (int i = threadIdx.x; i < a.rope_dims / 2; i += kPoolThreads)
    inv_freq[i] = rowprep::inv_freq(a.theta, i, a.rope_dims);
  __syncthreads();
  griddep_enter();

  constexpr int kEpc = 8 / kSplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = warp % kSplit;
  const int b = blockIdx.y;
  const int C = a.C;
  const int S = a.overlap ? 2 * a.m : a.m;
  const int own_lo = a.overlap ? a.m : 0;  // slots of the entry's own group
  const bool stream = a.pos != nullptr;
  const int E = a.T / a.m;
  int j, tok_ring = 0;
  bool active, has_entry;
  if (stream) {  // uniform over the CTA
    const int pos = a.pos[b];
    if (pos < 0 || (pos + 1) % a.m != 0) return;  // no group completes at this token
    j = (pos + 1) / a.m - 1;
    if (j >= a.E_max) {
      if (threadIdx.x == 0) atomicExch(a.err, CSA_DEVERR_INDEX);
      return;
    }
    tok_ring = pos - S + 1;  // token of ring row 0
    active = warp < kSplit;
    has_entry = true;
  } else {
    j = blockIdx.x * kEpc + warp / kSplit;
    const int groups = a.window != nullptr ? (a.T + a.m - 1) / a.m : E;
    active = j < groups;
    has_entry = j < E && (a.entries != nullptr || a.fp4 != nullptr);
  }
  const bool pooling = active && has_entry;
  const bool want_window = active && !stream && a.window != nullptr;
  const int first = a.overlap ? a.m * (j - 1) : a.m * j;  // token of slot 0
  const int per = (S + kSplit - 1) / kSplit;
  const int s_lo = sp * per, s_hi = min(S, s_lo + per);
  const size_t row_bytes = static_cast<size_t>(C) * (kBf16 ? 2 : 4);
  const uint8_t* kv = static_cast<const uint8_t*>(a.kv);
  const uint8_t* zl = static_cast<const uint8_t*>(a.logits);

  float mx[CPT], den[CPT], num[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    mx[e] = -INFINITY;
    den[e] = 0.f;
    num[e] = 0.f;
  }
  if (active && (pooling || want_window)) {
    constexpr int kPoolChunk = pool_chunk<RowBits<kBf16, CPT>::kWords>();
    for (int s0 = s_lo; s0 < s_hi; s0 += kPoolChunk) {
      RowBits<kBf16, CPT> xk[kPoolChunk], xz[kPoolChunk];
      bool ok[kPoolChunk];
      // every row of the chunk in flight before any is used
#pragma unroll
      for (int u = 0; u < kPoolChunk; ++u) {
        const int s = s0 + u;
        const int tok = first + s;
        ok[u] = s < s_hi && tok >= 0 && (stream || tok < a.T);
        const bool needed = ok[u] && (pooling || (want_window && s >= own_lo));
        ok[u] = needed;
        if (needed) {
          const size_t row = stream ? static_cast<size_t>(b) * S + (tok - tok_ring) : static_cast<size_t>(b) * a.T + tok;
          xk[u].load(kv + row * row_bytes, lane);
          if (pooling) xz[u].load(zl + row * row_bytes, lane);
        } else {
          xk[u].zero();  // weighted by 2^-inf = 0 in the chunk's softmax: must be a number
        }
      }
      bool any = false;
#pragma unroll
      for (int u = 0; u < kPoolChunk; ++u) any |= ok[u];
      if (pooling && any) {  // uniform over the warp
        // the chunk's slots at once: one rescale of the running state, then one exponential
        // per slot (rather than an online update per slot)
#pragma unroll
        for (int e = 0; e < CPT; e += 2) {
          float a0[kPoolChunk], a1[kPoolChunk];
          float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
          for (int u = 0; u < kPoolChunk; ++u) {
            const float2 bs = ok[u] ? __ldg(reinterpret_cast<const float2*>(a.bias + static_cast<size_t>(s0 + u) * C +
                                                                           lane * CPT + e))
                                    : make_float2(0.f, 0.f);
            a0[u] = ok[u] ? (xz[u].get(e) + bs.x) * kLog2e : -INFINITY;
            a1[u] = ok[u] ? (xz[u].get(e + 1) + bs.y) * kLog2e : -INFINITY;
            c0 = fmaxf(c0, a0[u]);
            c1 = fmaxf(c1, a1[u]);
          }
          softmax_chunk<kPoolChunk>(a0, xk, e, c0, mx[e], den[e], num[e]);
          softmax_chunk<kPoolChunk>(a1, xk, e + 1, c1, mx[e + 1], den[e + 1], num[e + 1]);
        }
      }
#pragma unroll
      for (int u = 0; u < kPoolChunk; ++u) {
        if (!ok[u]) continue;  // uniform over the warp
        const int s = s0 + u;
        if (want_window && s >= own_lo) {  // this token's window row, while it is in registers
          const int tok = first + s;
          float v[CPT];
#pragma unroll
          for (int e = 0; e < CPT; ++e) v[e] = xk[u].get(e);
          norm_rope_store<CPT>(v, lane, C, a.norm, a.eps, a.rope_dims, static_cast<double>(tok), inv_freq,
                               a.window + (static_cast<size_t>(b) * a.T + tok) * C);
        }
      }
    }
  }

  if constexpr (kSplit > 1) {
    // merge the warps' partial softmax states of the CTA's one entry (uniform branch)
    if (pooling) {
#pragma unroll
      for (int e = 0; e < CPT; ++e) {
        const int c = lane * CPT + e;
        part[(sp * 3 + 0) * C + c] = mx[e];
        part[(sp * 3 + 1) * C + c] = den[e];
        part[(sp * 3 + 2) * C + c] = num[e];
      }
    }
    __syncthreads();
    if (!pooling || sp != 0) return;
#pragma unroll
    for (int e = 0; e < CPT; ++e) {
      const int c = lane * CPT + e;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kSplit; ++w) M = fmaxf(M, part[(w * 3) * C + c]);
      float dn = 0.f, nm = 0.f;
#pragma unroll
      for (int w = 0; w < kSplit; ++w) {
        const float mw = part[(w * 3) * C + c];
        if (mw == -INFINITY) continue;  // a part without any slot
        const float r = fast_exp2(mw - M);
        dn = fmaf(part[(w * 3 + 1) * C + c], r, dn);
        nm = fmaf(part[(w * 3 + 2) * C + c], r, nm);
      }
      den[e] = dn;
      num[e] = nm;
    }
  }
  if (!pooling) return;

  float v[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) v[e] = __fdividef(num[e], den[e]);  // den >= 1
  const size_t erow = static_cast<size_t>(b) * a.E_max + j;
  if (a.fp4 != nullptr)  // indexer key cache: pooled values before norm / RoPE
    fp4_store<CPT>(v, lane, a.fp4 + erow * (C / 2), a.fp4_scale + erow * (C / 32));
  if (a.entries != nullptr)
    norm_rope_store<CPT>(v, lane, C, a.norm, a.eps, a.rope_dims, static_cast<double>(a.m) * (j + 1) - 1.0, inv_freq,
                         a.entries + erow * C);
}

// One CTA per row (all heads at that row's position); warp w takes heads w, w + 8, ...,
// two at a time (both rows' loads in flight before either is used).
template <bool kBf16, int CPT>
__global__ void __launch_bounds__(kPoolThreads) norm_rope_kernel(NormRopeArgs a) {
  extern __shared__ __align__(16) uint8_t nr_smem[];
  double* inv_freq = reinterpret_cast<double*>(nr_smem);
  for (int i = threadIdx.x; i < a.rope_dims / 2; i += blockDim.x)
    inv_freq[i] = rowprep::inv_freq(a.theta, i, a.rope_dims);
  __syncthreads();
  griddep_enter();
  const int64_t row = blockIdx.x;
  const int C = a.C;
  const double pos = static_cast<double>(a.pos ? static_cast<int64_t>(a.pos[row]) : row % a.pos_mod);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const size_t row_bytes = static_cast<size_t>(C) * (kBf16 ? 2 : 4);
  const uint8_t* x = static_cast<const uint8_t*>(a.x);
  for (int h0 = warp; h0 < a.heads; h0 += 2 * nw) {
    const int h1 = h0 + nw;
    RowBits<kBf16, CPT> r0, r1;
    const size_t v0 = static_cast<size_t>(row) * a.heads + h0;
    r0.load(x + v0 * row_bytes, lane);
    if (h1 < a.heads) r1.load(x + (v0 + nw) * row_bytes, lane);
    float v[CPT];
#pragma unroll
    for (int e = 0; e < CPT; ++e) v[e] = r0.get(e);
    norm_rope_store<CPT>(v, lane, C, a.norm, a.eps, a.rope_dims, pos, inv_freq, a.out + v0 * C);
    if (h1 < a.heads) {
#pragma unroll
      for (int e = 0; e < CPT; ++e) v[e] = r1.get(e);
      norm_rope_store<CPT>(v, lane, C, a.norm, a.eps, a.rope_dims, pos, inv_freq, a.out + (v0 + nw) * C);
    }
  }
}

template <bool kBf16, int CPT>
cudaError_t launch_norm_rope_t(const NormRopeArgs& a, cudaStream_t s) {
  const int warps = a.heads < 8 ? a.heads : 8;
  const dim3 grid(static_cast<unsigned>(a.rows)), block(32 * warps);
  const size_t smem = sizeof(double) * (a.rope_dims / 2 > 0 ? a.rope_dims / 2 : 1);
  return launch_pdl(norm_rope_kernel<kBf16, CPT>, grid, block, smem, s, a);
}

template <bool kBf16>
cudaError_t launch_norm_rope_c(const NormRopeArgs& a, cudaStream_t s) {
  switch (a.C / 32) {
    case 2: return launch_norm_rope_t<kBf16, 2>(a, s);
    case 4: return launch_norm_rope_t<kBf16, 4>(a, s);
    case 8: return launch_norm_rope_t<kBf16, 8>(a, s);
    case 16: return launch_norm_rope_t<kBf16, 16>(a, s);
    case 32: return launch_norm_rope_t<kBf16, 32>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool kBf16, int CPT, int kSplit>
cudaError_t launch_pool_t(const PoolArgs& a, cudaStream_t s) {
  const size_t smem = pool_smem_bytes(a.C, a.rope_dims, kSplit);
  static int attr_set[64];
  const cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(pool_kernel<kBf16, CPT, kSplit>), smem, attr_set);
  if (e != cudaSuccess) return e;
  if (a.pos != nullptr) return launch_pdl(pool_kernel<kBf16, CPT, kSplit>, dim3(1, a.B), dim3(kPoolThreads), smem, s, a);
  const int groups = a.window != nullptr ? (a.T + a.m - 1) / a.m : a.T / a.m;
  constexpr int kEpc = 8 / kSplit;
  const dim3 grid((groups + kEpc - 1) / kEpc, a.B);
  return launch_pdl(pool_kernel<kBf16, CPT, kSplit>, grid, dim3(kPoolThreads), smem, s, a);
}

template <bool kBf16, int kSplit>
cudaError_t launch_pool_c(const PoolArgs& a, cudaStream_t s) {
  switch (a.C / 32) {
    case 2: return launch_pool_t<kBf16, 2, kSplit>(a, s);
    case 4: return launch_pool_t<kBf16, 4, kSplit>(a, s);
    case 8: return launch_pool_t<kBf16, 8, kSplit>(a, s);
    case 16: return launch_pool_t<kBf16, 16, kSplit>(a, s);
    case 32: return launch_pool_t<kBf16, 32, kSplit>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  return a.in_bf16 ? launch_norm_rope_c<true>(a, s) : launch_norm_rope_c<false>(a, s);
}

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s) {
  if (a.entries == nullptr && a.fp4 == nullptr && a.window == nullptr) return cudaSuccess;
  if (a.pos == nullptr && (a.window != nullptr ? a.T : a.T / a.m) == 0) return cudaSuccess;
  // eight warps per entry once an entry has at least 64 slots (HCA), else one
  const int S = (a.overlap ? 2 : 1) * a.m;
  const bool split = S >= 64;
  if (a.in_bf16) return split ? launch_pool_c<true, 8>(a, s) : launch_pool_c<true, 1>(a, s);
  return split ? launch_pool_c<false, 8>(a, s) : launch_pool_c<false, 1>(a, s);
}

}  // namespace csa
