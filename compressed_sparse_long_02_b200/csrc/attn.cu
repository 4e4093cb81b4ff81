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
constexpr int kAttnThreads = 416;  // 8 softmax warps, 4 gather warps, 1 MMA warp
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kSplitSMs = 148;            // B200 SM count used to size decode splits

constexpr size_t kOffQ = 0;                      // 64 KB: [8 d-atoms][64 heads][128 B]
constexpr size_t kOffKV = 64 * 1024;             // 128 KB: [8 d-atoms][128 keys][128 B]
constexpr size_t kOffP = kOffKV + 128 * 1024;    // 16 KB: [128 keys][128 B]
constexpr size_t kOffSmall = kOffP + 16 * 1024;  // reductions, running stats, barriers
constexpr size_t kOffIdx = kOffSmall + 4096;     // 8 KB: this CTA's slice of the index list
constexpr int kIdxCap = 2048;
constexpr size_t kAttnSmem = kOffIdx + 4 * kIdxCap + 1024;
constexpr int kSlabLag = 3;  // cp.async groups (16 KB slabs) a producer keeps in flight

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

// 32 per-thread values (one per head) reduced over the 32 lanes of the warp; on return
// v[0] holds the warp total of head `lane`.
template <bool kMax>
__device__ __forceinline__ void xreduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int off = 16 >> lvl;
    const int half = 16 >> lvl;
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
  CSA_TB(0);
  griddep_enter();
  CSA_TB(1);
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
  uint64_t* slab_full = bars + 1;   // [8]: 16 KB slab (64 of the 512 dims) of the current tile loaded
  uint64_t* slab_free = bars + 9;   // [8]: the MMAs reading that slab have completed
  uint64_t* s_full = bars + 17;
  uint64_t* p_full = bars + 18;
  uint64_t* o_done = bars + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + kOffIdx);
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
    for (int i = 0; i < 8; ++i) {
      mbar_init(&slab_full[i], 128);
      mbar_init(&slab_free[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kH) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int tslot = blockIdx.x < 2 ? 4 + static_cast<int>(blockIdx.x) : -1;
  if (threadIdx.x == 0) CSA_T(tslot, 0);
  CSA_TB(2);

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------ gather producers
    const int pw = warp - 8;
    const int ptid = threadIdx.x - 256;
    // this CTA's slice of the index list, staged once (no dependent global load per tile)
    const int sel_here = max(0, min(row_end, kl.n_sel) - row_begin);
    const bool staged = !p.dense && sel_here <= kIdxCap;
    if (staged)
      for (int i = ptid; i < sel_here; i += 128) sidx[i] = p.idx[static_cast<size_t>(n) * p.k + row_begin + i];
    named_bar_sync(2, 128);
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
      if (ptid == 0) CSA_T(tslot, 1);
    }
    bool ok = true;
    for (int it = 0; ok && it < n_tiles; ++it) {
      // slab 0 of the previous tile is free only after the softmax of that tile has
      // arrived on p_full, i.e. after it read row_ok: row_ok may be rewritten now
      if (it > 0 && !warp_wait(&slab_free[0], (it - 1) & 1, p.err, abort_flag)) break;
      // each lane resolves the source of one of this warp's 32 rows
      const int r_own = pw * 32 + lane;
      const int g = row_begin + it * kBN + r_own;
      const uint16_t* src = p.entries;
      bool valid = false;
      if (g < row_end) {
        if (g < kl.n_sel) {
          const int e = p.dense ? g : (staged ? sidx[g - row_begin] : p.idx[static_cast<size_t>(n) * p.k + g]);
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
      row_ok[r_own] = valid ? 1 : 0;  // read by the softmax after it observes slab_full[7]
      const unsigned long long src_ll = reinterpret_cast<unsigned long long>(src);
      // slab by slab (64 dims x 128 rows = 16 KB): each instruction moves 4 rows x 128 B
      for (int ka = 0; ka < 8; ++ka) {
        if (it > 0 && ka > 0 && !warp_wait(&slab_free[ka], (it - 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int rr = 0; rr < 32; rr += 4) {
          const int rl = rr + (lane >> 3);
          const uint16_t* rs = reinterpret_cast<const uint16_t*>(__shfl_sync(0xffffffffu, src_ll, rl));
          const bool rv = __shfl_sync(0xffffffffu, valid, rl);
          const int c = lane & 7;
          cp_async_16(smem_u32(sKV + ka * 16384) + sw128(pw * 32 + rl, c), rs + (ka * 8 + c) * 8, rv);
        }
        cp_async_commit();
        if (ka >= kSlabLag) {
          cp_async_wait_group<kSlabLag>();
          fence_proxy_async_smem();
          mbar_arrive(&slab_full[ka - kSlabLag]);
        }
      }
      if (ptid == 0 && it < 8) CSA_T(tslot, 8 + it);
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      if (ptid == 0 && it < 8) CSA_T(tslot, 16 + it);
      if (ok)
        for (int ka = 8 - kSlabLag; ka < 8; ++ka) mbar_arrive(&slab_full[ka]);
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, kH, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, kH, true, true);
    const uint32_t q0 = smem_u32(sQ), kv0 = smem_u32(sKV), p0 = smem_u32(sP);
    bool ok = warp_wait(q_full, 0, p.err, abort_flag);
    for (int it = 0; ok && it < n_tiles; ++it) {
      // S^T = K Q^T, slab by slab as the slabs arrive
      for (int ka = 0; ka < 8; ++ka) {
        if (!warp_wait(&slab_full[ka], it & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColS, smem_desc(kv0 + ka * 16384 + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(q0 + ka * 8192 + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, (ka | kk) ? 1u : 0u);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(s_full);
      if (lane == 0 && it < 8) CSA_T(tslot, 24 + it);
      __syncwarp();
      if (!warp_wait(p_full, it & 1, p.err, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        // O^T += V^T P^T; each 128-dim chunk frees its two slabs as soon as its MMAs retire
#pragma unroll 1
        for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + kColO + 64 * dc, smem_desc(kv0 + 2 * dc * 16384 + ks * 2048, 16384, 1024, kSwizzle128B),
                     smem_desc(p0 + ks * 2048, 16384, 1024, kSwizzle128B), idesc_pv, (it > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&slab_free[2 * dc]);
          tc_commit(&slab_free[2 * dc + 1]);
        }
        tc_commit(o_done);
        if (it < 8) CSA_T(tslot, 32 + it);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    // thread = one key row of the tile (TMEM lane 32*(warp%4)+lane) and 32 heads
    // (hh = warp/4 selects heads 0-31 or 32-63).  Sums over keys stay per thread in
    // registers and are reduced once at the end; the running max is reduced only on the
    // first tile or when a logit exceeds it by more than 2^8 (then O^T is rescaled).
    const int q4 = warp & 3, hh = warp >> 2;
    const int t = 32 * q4 + lane;
    const int h0 = 32 * hh;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    float lacc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) lacc[i] = 0.f;
    for (int it = 0; it < n_tiles; ++it) {
      const bool got_s = mbar_wait(s_full, it & 1, p.err, abort_flag);
      if (named_bar_or(1, 256, !got_s)) break;  // the group leaves together
      if (t == 0 && hh == 0 && it < 8) CSA_T(tslot, 40 + it);
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld16(tmem + lane_base + kColS + h0, sr);
      tmem_ld16(tmem + lane_base + kColS + h0 + 16, sr + 16);
      tmem_wait_ld();
      // every producer wrote row_ok before arriving on slab_full[7] of this tile
      const bool got_kv = mbar_wait(&slab_full[7], it & 1, p.err, abort_flag);
      if (named_bar_or(1, 256, !got_kv)) break;
      const bool valid = row_begin + it * kBN + t < row_end && row_ok[t] != 0;
      float x[32];
      bool over = false;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 mm = *reinterpret_cast<const float4*>(m_run + h0 + i);
        const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x[i + j] = valid ? __uint_as_float(sr[i + j]) * p.scale_log2 : -INFINITY;
          over |= x[i + j] > mv[j] + kRescaleThreshold;
        }
      }
      const bool move_max = named_bar_or(1, 256, over);  // always true on the first tile
      if (move_max) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = x[i];
        xreduce32<true>(v);
        red_max[q4 * 64 + h0 + lane] = v[0];
        named_bar_sync(1, 256);
        if (threadIdx.x < kH) {
          const int h = threadIdx.x;
          const float tm = fmaxf(fmaxf(red_max[h], red_max[64 + h]), fmaxf(red_max[128 + h], red_max[192 + h]));
          const float mo = m_run[h];
          const float mn = fmaxf(mo, tm);
          alpha[h] = mo == -INFINITY ? 0.f : exp2f(mo - mn);
          m_run[h] = mn;
        }
        named_bar_sync(1, 256);
#pragma unroll
        for (int i = 0; i < 32; ++i) lacc[i] *= alpha[h0 + i];
      }
      float pr[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 mm = *reinterpret_cast<const float4*>(m_run + h0 + i);
        pr[i] = valid ? exp2f(x[i] - mm.x) : 0.f;
        pr[i + 1] = valid ? exp2f(x[i + 1] - mm.y) : 0.f;
        pr[i + 2] = valid ? exp2f(x[i + 2] - mm.z) : 0.f;
        pr[i + 3] = valid ? exp2f(x[i + 3] - mm.w) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) lacc[i] += pr[i];
      // the P buffer and O^T are still in use by the previous tile's PV MMAs
      const bool got_o = it == 0 || mbar_wait(o_done, (it - 1) & 1, p.err, abort_flag);
      if (named_bar_or(1, 256, !got_o)) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w4 = make_uint4(pack_bf16x2(pr[8 * c], pr[8 * c + 1]), pack_bf16x2(pr[8 * c + 2], pr[8 * c + 3]),
                                    pack_bf16x2(pr[8 * c + 4], pr[8 * c + 5]), pack_bf16x2(pr[8 * c + 6], pr[8 * c + 7]));
        *reinterpret_cast<uint4*>(sP + sw128(t, 4 * hh + c)) = w4;
      }
      if (move_max && it > 0) {  // move this warp's O^T columns (heads h0..h0+31) to the new max
#pragma unroll 1
        for (int dc = 0; dc < 4; ++dc) {
          uint32_t o[32];
          const uint32_t ta = tmem + lane_base + kColO + 64 * dc + h0;
          tmem_ld16(ta, o);
          tmem_ld16(ta + 16, o + 16);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[h0 + i]);
          tmem_st16(ta, o);
          tmem_st16(ta + 16, o + 16);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (t == 0 && hh == 0 && it < 8) CSA_T(tslot, 48 + it);
    }
    // ------------------------------------------------------------ epilogue
    const bool ok = !named_bar_or(1, 256, !mbar_wait(o_done, (n_tiles - 1) & 1, p.err, abort_flag));
    if (t == 0 && hh == 0) CSA_T(tslot, 2);
    tc_fence_after();
    xreduce32<false>(lacc);  // lane holds head h0+lane summed over this warp's 32 keys
    red_sum[q4 * 64 + h0 + lane] = lacc[0];
    named_bar_sync(1, 256);
    if (threadIdx.x < kH) {
      const int h = threadIdx.x;
      l_run[h] = (red_sum[h] + red_sum[64 + h]) + (red_sum[128 + h] + red_sum[192 + h]);
      inv_l[h] = l_run[h] > 0.f ? 1.0f / l_run[h] : 0.f;
    }
    named_bar_sync(1, 256);
    if (ok) {
#pragma unroll 1
      for (int dc = 0; dc < 4; ++dc) {
        uint32_t o[32];
        const uint32_t ta = tmem + lane_base + kColO + 64 * dc + h0;
        tmem_ld16(ta, o);
        tmem_ld16(ta + 16, o + 16);
        tmem_wait_ld();
        const int d = dc * 128 + t;
        if (p.splits == 1) {
          uint16_t* ob = p.out + (static_cast<size_t>(n) * kH + h0) * kD + d;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(o[i]) * inv_l[h0 + i]);
            ob[i * kD] = *reinterpret_cast<const uint16_t*>(&bv);
          }
        } else {
          float* pb = p.part_o + ((static_cast<size_t>(n) * p.splits + split) * kH + h0) * kD + d;
#pragma unroll
          for (int i = 0; i < 32; ++i) pb[i * kD] = __uint_as_float(o[i]);
        }
      }
      if (threadIdx.x < kH) {
        const int h = threadIdx.x;
        if (p.splits == 1) {
          if (p.lse) p.lse[n * kH + h] = (m_run[h] + log2f(l_run[h])) * 0.69314718055994531f;
        } else {
          p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + h] = make_float2(m_run[h], l_run[h]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) CSA_T(tslot, 3);
  CSA_TB(3);
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// one warp per (query, head): combine the split partials
__global__ void attn_merge_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml, int Nq,
                                  int splits, uint16_t* __restrict__ out, float* __restrict__ lse) {
  griddep_enter();
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
  p.splits = splits;
  p.rows_per_split = std::max(32, (((max_keys + splits - 1) / splits) + 31) / 32 * 32);
  if (splits > 1) {
    const size_t o_bytes = static_cast<size_t>(a.Nq) * splits * kH * kD * sizeof(float);
    uintptr_t base = reinterpret_cast<uintptr_t>(a.ws);
    base = (base + 255) & ~uintptr_t(255);
    p.part_o = reinterpret_cast<float*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + o_bytes);
  }
  cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(attn_kernel), kAttnSmem, g_attn_smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(attn_kernel, dim3(a.Nq * splits), dim3(kAttnThreads), kAttnSmem, s, p);
  if (e != cudaSuccess || splits == 1) return e;
  const int warps = a.Nq * kH;
  return launch_pdl(attn_merge_kernel, dim3((warps * 32 + 255) / 256), dim3(256), 0, s,
                    static_cast<const float*>(p.part_o), static_cast<const float2*>(p.part_ml), a.Nq, splits, a.out, a.lse);
}

}  // namespace csa
