// attn.cu -- core shared-KV multi-query attention over (selected entries | all visible
// entries) plus the raw-token sliding window, on tcgen05 tensor cores.
//
// Sources: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence"
// section 2.3 (shared-KV MQA over the k selected entries; HCA attends densely);
// "DeepSeek-V4: Million-Token Context" CSA and HCA stages (each head attends to the
// picked set plus a sliding window of recent tokens); "Follow the white rabbit"
// (window of the most recent 128 tokens, covering the unfinished group).
//
// All H = 64 heads of one query share one key list, so a CTA works on one query
// (or a contiguous split of its key list) and puts KEYS on the MMA M axis:
//   S^T[128 keys, 64 heads]  = K[128 x 512] . Q^T           (K-major A and B, SW128)
//   O^T[512 d, 64 heads]    += V^T[512 x 128] . P^T         (the same smem tile read
//                                                            MN-major, P^T MN-major)
// with K = V (shared KV).  S^T takes 64 TMEM columns, O^T 4 x 64.  Softmax runs one
// thread per key (TMEM lane): head maxima and sums over keys are reduced with a
// shuffle transpose-reduce (62 shuffles for 64 heads) and a 4-warp smem step.  The
// running max is only moved when a tile raises it by more than 2^8, so O^T rarely
// needs a rescale in TMEM.  Rows are gathered with cp.async (16-byte chunks, coalesced
// 512-byte runs per warp) straight into the SWIZZLE_128B layout.
//
// Roles (288 threads): warps 0-3 softmax + epilogue, warps 4-7 gather producers,
// warp 8 TMEM owner and MMA issuer.  When a query's keys are split over several CTAs
// (decode), each CTA writes an unnormalised fp32 partial and (max, sum); a merge
// kernel combines them.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace csa {
namespace {

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kBN = 128;  // keys per tile
constexpr int kAttnThreads = 288;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kSplitSMs = 148;            // B200 SM count used to size decode splits

constexpr size_t kOffQ = 0;                      // 64 KB: [8 d-atoms][64 heads][128 B]
constexpr size_t kOffKV = 64 * 1024;             // 128 KB: [8 d-atoms][128 keys][128 B]
constexpr size_t kOffP = kOffKV + 128 * 1024;    // 16 KB: [128 keys][128 B]
constexpr size_t kOffSmall = kOffP + 16 * 1024;  // reductions, running stats, barriers
constexpr size_t kAttnSmem = kOffSmall + 4096 + 1024;

struct AttnParams {
  int Nq, k, W, B, E_max, Tw, mprime, dense;
  float scale_log2;
  const uint16_t* q;
  const int32_t* q_pos;
  const int32_t* q_seq;
  const uint16_t* entries;
  const int32_t* idx;
  const int32_t* cnt;
  const int32_t* n_entries;
  const uint16_t* window;
  const int32_t* window_base;
  uint16_t* out;
  float* lse;
  float* part_o;   // [Nq, splits, H, D]
  float2* part_ml; // [Nq, splits, H]
  int rows_per_split, splits;
  int32_t* err;
};

struct KeyList {
  int b, n_sel, n_win;
  int64_t u_lo, wbase;
};

__device__ __forceinline__ KeyList key_list(const AttnParams& p, int n) {
  KeyList kl;
  kl.b = p.q_seq[n];
  const int64_t t = p.q_pos[n];
  if (p.dense) {
    int64_t v = (t + 1) / p.mprime;
    v = v < 0 ? 0 : v;
    const int64_t ne = min(p.n_entries[kl.b], p.E_max);
    kl.n_sel = static_cast<int>(v < ne ? v : ne);
  } else {
    const int c = p.cnt ? p.cnt[n] : 0;
    kl.n_sel = c < 0 ? 0 : (c > p.k ? p.k : c);
  }
  kl.wbase = p.window_base[kl.b];
  int64_t lo = t - p.W + 1;
  if (lo < 0) lo = 0;
  if (lo < kl.wbase) lo = kl.wbase;
  int64_t hi = t;
  if (hi > kl.wbase + p.Tw - 1) hi = kl.wbase + p.Tw - 1;
  kl.u_lo = lo;
  kl.n_win = (p.W > 0 && hi >= lo) ? static_cast<int>(hi - lo + 1) : 0;
  return kl;
}

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {  // byte offset inside an 8-row x 128 B atom column
  return static_cast<uint32_t>(row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// 64 per-thread values (one per head) reduced over the 32 lanes of the warp; on
// return v[0], v[1] hold the warp totals of heads 2*lane and 2*lane+1.
template <bool kMax>
__device__ __forceinline__ void xreduce64(float (&v)[64]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int off = 16 >> lvl;
    const int half = 32 >> lvl;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  float* red_max = reinterpret_cast<float*>(smem + kOffSmall);  // [4][64]
  float* red_sum = red_max + 256;                                // [4][64]
  float* m_run = red_sum + 256;                                  // [64]
  float* l_run = m_run + 64;                                // [64]
  float* alpha = l_run + 64;                                // [64]
  float* inv_l = alpha + 64;                                // [64]
  uint8_t* row_ok = reinterpret_cast<uint8_t*>(inv_l + 64); // [128]: key row holds a valid source
  uint64_t* bars = reinterpret_cast<uint64_t*>(row_ok + 128);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;
  uint64_t* s_full = bars + 2;
  uint64_t* p_full = bars + 3;
  uint64_t* o_done = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int n = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.q_seq[n] < 0 || p.q_seq[n] >= p.B) {
    if (threadIdx.x == 0) atomicExch(p.err, CSA_DEVERR_INDEX);
    return;
  }
  const KeyList kl = key_list(p, n);
  const int nk = kl.n_sel + kl.n_win;
  const int row_begin = split * p.rows_per_split;
  const int row_end = min(nk, row_begin + p.rows_per_split);
  const int n_tiles = row_end > row_begin ? (row_end - row_begin + kBN - 1) / kBN : 0;

  if (n_tiles == 0) {  // nothing to attend to in this split
    if (p.splits == 1) {
      for (int i = threadIdx.x; i < kH * kD / 2; i += blockDim.x)
        reinterpret_cast<uint32_t*>(p.out + static_cast<size_t>(n) * kH * kD)[i] = 0u;
      if (p.lse && threadIdx.x < kH) p.lse[n * kH + threadIdx.x] = -INFINITY;
    } else if (threadIdx.x < kH) {
      p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + threadIdx.x] = make_float2(-INFINITY, 0.f);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(kv_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kH) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ gather producers
    const int pw = warp - 4;
    {  // query: 64 head rows of 1 KB
      const uint16_t* qb = p.q + static_cast<size_t>(n) * kH * kD;
      for (int h = pw * 16; h < pw * 16 + 16; ++h) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c = lane + 32 * half;
          cp_async_16(smem_u32(sQ + (c >> 3) * 8192) + sw128(h, c), qb + h * kD + c * 8, true);
        }
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
    for (int it = 0; it < n_tiles; ++it) {
      if (it > 0 && !warp_wait(o_done, (it - 1) & 1, p.err, abort_flag)) break;
      // each lane resolves the source of one of this warp's 32 rows
      const int r_own = pw * 32 + lane;
      const int g = row_begin + it * kBN + r_own;
      const uint16_t* src = p.entries;
      bool valid = false;
      if (g < row_end) {
        if (g < kl.n_sel) {
          const int e = p.dense ? g : p.idx[static_cast<size_t>(n) * p.k + g];
          if (e >= 0 && e < p.E_max) {
            src = p.entries + (static_cast<size_t>(kl.b) * p.E_max + e) * kD;
            valid = true;
          } else {
            atomicExch(p.err, CSA_DEVERR_INDEX);
          }
        } else {
          const int64_t u = kl.u_lo + (g - kl.n_sel);
          src = p.window + (static_cast<size_t>(kl.b) * p.Tw + static_cast<size_t>(u - kl.wbase)) * kD;
          valid = true;
        }
      }
      row_ok[r_own] = valid ? 1 : 0;  // read by the softmax after it observes kv_full
      const unsigned long long src_ll = reinterpret_cast<unsigned long long>(src);
      for (int rr = 0; rr < 32; ++rr) {
        const int r = pw * 32 + rr;
        const uint16_t* rs = reinterpret_cast<const uint16_t*>(__shfl_sync(0xffffffffu, src_ll, rr));
        const bool rv = __shfl_sync(0xffffffffu, valid, rr);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c = lane + 32 * half;
          cp_async_16(smem_u32(sKV + (c >> 3) * 16384) + sw128(r, c), rs + c * 8, rv);
        }
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(kv_full);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, kH, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, kH, true, true);
    const uint32_t q0 = smem_u32(sQ), kv0 = smem_u32(sKV), p0 = smem_u32(sP);
    bool ok = warp_wait(q_full, 0, p.err, abort_flag);
    for (int it = 0; ok && it < n_tiles; ++it) {
      if (!warp_wait(kv_full, it & 1, p.err, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll 1
        for (int ka = 0; ka < 8; ++ka)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColS, smem_desc(kv0 + ka * 16384 + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(q0 + ka * 8192 + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, (ka | kk) ? 1u : 0u);
        tc_commit(s_full);
      }
      __syncwarp();
      if (!warp_wait(p_full, it & 1, p.err, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll 1
        for (int dc = 0; dc < 4; ++dc)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + kColO + 64 * dc, smem_desc(kv0 + 2 * dc * 16384 + ks * 2048, 16384, 1024, kSwizzle128B),
                     smem_desc(p0 + ks * 2048, 16384, 1024, kSwizzle128B), idesc_pv, (it > 0 || ks > 0) ? 1u : 0u);
        tc_commit(o_done);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int t = threadIdx.x;  // key row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    for (int it = 0; it < n_tiles; ++it) {
      const bool got_s = mbar_wait(s_full, it & 1, p.err, abort_flag);
      if (named_bar_or(1, 128, !got_s)) break;  // the group leaves together
      tc_fence_after();
      uint32_t sr[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(tmem + lane_base + kColS + 16 * c, sr + 16 * c);
      tmem_wait_ld();
      // kv_full of this tile completed before s_full; waiting on it orders the row_ok writes
      const bool got_kv = mbar_wait(kv_full, it & 1, p.err, abort_flag);
      if (named_bar_or(1, 128, !got_kv)) break;
      const bool valid = row_begin + it * kBN + t < row_end && row_ok[t] != 0;
      float x[64], v[64];
#pragma unroll
      for (int h = 0; h < 64; ++h) {
        x[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
        v[h] = x[h];
      }
      xreduce64<true>(v);
      red_max[warp * 64 + 2 * lane] = v[0];
      red_max[warp * 64 + 2 * lane + 1] = v[1];
      named_bar_sync(1, 128);
      bool need = false;
      if (t < kH) {
        const float tm = fmaxf(fmaxf(red_max[t], red_max[64 + t]), fmaxf(red_max[128 + t], red_max[192 + t]));
        const float mo = m_run[t];
        float mn = mo, al = 1.f;
        if (mo == -INFINITY) {
          mn = tm;
        } else if (tm > mo + kRescaleThreshold) {
          mn = tm;
          al = exp2f(mo - mn);
          need = true;
        }
        m_run[t] = mn;
        alpha[t] = al;
      }
      const bool any_rescale = named_bar_or(1, 128, need);
      // probabilities (relative to the running max) and their per-head sums
      float pr[64];
#pragma unroll
      for (int h = 0; h < 64; h += 4) {
        const float4 mm = *reinterpret_cast<const float4*>(m_run + h);
        pr[h] = valid ? exp2f(x[h] - mm.x) : 0.f;
        pr[h + 1] = valid ? exp2f(x[h + 1] - mm.y) : 0.f;
        pr[h + 2] = valid ? exp2f(x[h + 2] - mm.z) : 0.f;
        pr[h + 3] = valid ? exp2f(x[h + 3] - mm.w) : 0.f;
      }
#pragma unroll
      for (int h = 0; h < 64; ++h) v[h] = pr[h];
      xreduce64<false>(v);
      red_sum[warp * 64 + 2 * lane] = v[0];
      red_sum[warp * 64 + 2 * lane + 1] = v[1];
      // the P buffer and O^T are still in use by the previous tile's PV MMAs
      const bool got_o = it == 0 || mbar_wait(o_done, (it - 1) & 1, p.err, abort_flag);
      if (named_bar_or(1, 128, !got_o)) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w4 = make_uint4(pack_bf16x2(pr[8 * c], pr[8 * c + 1]), pack_bf16x2(pr[8 * c + 2], pr[8 * c + 3]),
                                    pack_bf16x2(pr[8 * c + 4], pr[8 * c + 5]), pack_bf16x2(pr[8 * c + 6], pr[8 * c + 7]));
        *reinterpret_cast<uint4*>(sP + sw128(t, c)) = w4;
      }
      if (any_rescale) {  // move the O^T columns (heads) to the new running max
#pragma unroll 1
        for (int dc = 0; dc < 4; ++dc) {
          uint32_t o[64];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld16(tmem + lane_base + kColO + 64 * dc + 16 * c, o + 16 * c);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 64; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_st16(tmem + lane_base + kColO + 64 * dc + 16 * c, o + 16 * c);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      named_bar_sync(1, 128);
      if (t < kH)
        l_run[t] = l_run[t] * alpha[t] + ((red_sum[t] + red_sum[64 + t]) + (red_sum[128 + t] + red_sum[192 + t]));
    }
    // ------------------------------------------------------------ epilogue
    const bool ok = !named_bar_or(1, 128, !mbar_wait(o_done, (n_tiles - 1) & 1, p.err, abort_flag));
    tc_fence_after();
    if (t < kH) inv_l[t] = l_run[t] > 0.f ? 1.0f / l_run[t] : 0.f;
    named_bar_sync(1, 128);
    if (ok) {
#pragma unroll 1
      for (int dc = 0; dc < 4; ++dc) {
        uint32_t o[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tmem + lane_base + kColO + 64 * dc + 16 * c, o + 16 * c);
        tmem_wait_ld();
        const int d = dc * 128 + t;
        if (p.splits == 1) {
          uint16_t* ob = p.out + static_cast<size_t>(n) * kH * kD + d;
#pragma unroll
          for (int h = 0; h < 64; ++h) {
            const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(o[h]) * inv_l[h]);
            ob[h * kD] = *reinterpret_cast<const uint16_t*>(&b);
          }
        } else {
          float* pb = p.part_o + (static_cast<size_t>(n) * p.splits + split) * kH * kD + d;
#pragma unroll
          for (int h = 0; h < 64; ++h) pb[h * kD] = __uint_as_float(o[h]);
        }
      }
      if (t < kH) {
        if (p.splits == 1) {
          if (p.lse) p.lse[n * kH + t] = (m_run[t] + log2f(l_run[t])) * 0.69314718055994531f;
        } else {
          p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + t] = make_float2(m_run[t], l_run[t]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// one warp per (query, head): combine the split partials
__global__ void attn_merge_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml, int Nq,
                                  int splits, uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= Nq * kH) return;
  const int n = gw / kH, h = gw % kH;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const float2 ml = part_ml[(static_cast<size_t>(n) * splits + s) * kH + h];
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float2 ml = part_ml[(static_cast<size_t>(n) * splits + s) * kH + h];
    if (!(ml.y > 0.f)) continue;
    const float wgt = exp2f(ml.x - M);
    L = fmaf(ml.y, wgt, L);
    const float4* src =
        reinterpret_cast<const float4*>(part_o + ((static_cast<size_t>(n) * splits + s) * kH + h) * kD) + lane * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(src + i);
      acc[4 * i] = fmaf(v.x, wgt, acc[4 * i]);
      acc[4 * i + 1] = fmaf(v.y, wgt, acc[4 * i + 1]);
      acc[4 * i + 2] = fmaf(v.z, wgt, acc[4 * i + 2]);
      acc[4 * i + 3] = fmaf(v.w, wgt, acc[4 * i + 3]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint32_t* o = reinterpret_cast<uint32_t*>(out + (static_cast<size_t>(n) * kH + h) * kD + lane * 16);
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  if (lse && lane == 0) lse[n * kH + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

int g_attn_smem[64];

int split_count(int Nq, int max_keys) {
  const int tiles = std::max(1, (max_keys + kBN - 1) / kBN);
  if (Nq >= kSplitSMs) return 1;
  return std::max(1, std::min(tiles, kSplitSMs / std::max(1, Nq)));
}

}  // namespace

size_t attn_workspace_bytes(int Nq, int /*H*/, int /*D*/, int max_keys) {
  const int splits = split_count(Nq, max_keys);
  if (splits == 1) return 256;
  return static_cast<size_t>(Nq) * splits * kH * (kD * sizeof(float) + sizeof(float2)) + 512;
}

cudaError_t launch_attention(const AttnArgs& a, int max_keys, cudaStream_t s) {
  if (a.Nq == 0) return cudaSuccess;
  AttnParams p{};
  p.Nq = a.Nq;
  p.k = a.k;
  p.W = a.W;
  p.B = a.B;
  p.E_max = a.E_max;
  p.Tw = a.Tw;
  p.mprime = a.mprime;
  p.dense = a.dense;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.q = a.q;
  p.q_pos = a.q_pos;
  p.q_seq = a.q_seq;
  p.entries = a.entries;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.n_entries = a.n_entries;
  p.window = a.window;
  p.window_base = a.window_base;
  p.out = a.out;
  p.lse = a.lse;
  p.err = device_error_word();
  const int splits = split_count(a.Nq, max_keys);
  const int tiles = std::max(1, (max_keys + kBN - 1) / kBN);
  p.splits = splits;
  p.rows_per_split = ((tiles + splits - 1) / splits) * kBN;
  if (splits > 1) {
    const size_t o_bytes = static_cast<size_t>(a.Nq) * splits * kH * kD * sizeof(float);
    uintptr_t base = reinterpret_cast<uintptr_t>(a.ws);
    base = (base + 255) & ~uintptr_t(255);
    p.part_o = reinterpret_cast<float*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + o_bytes);
  }
  cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(attn_kernel), kAttnSmem, g_attn_smem);
  if (e != cudaSuccess) return e;
  attn_kernel<<<a.Nq * splits, kAttnThreads, kAttnSmem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int warps = a.Nq * kH;
  attn_merge_kernel<<<(warps * 32 + 255) / 256, 256, 0, s>>>(p.part_o, p.part_ml, a.Nq, splits, a.out, a.lse);
  return cudaGetLastError();
}

}  // namespace csa
