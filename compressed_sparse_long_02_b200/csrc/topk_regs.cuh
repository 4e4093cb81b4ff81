// topk_regs.cuh -- exact top-k of one query row held in registers by a thread-block
// cluster of C CTAs (C = 1: one CTA), shared by the stand-alone top-k kernel (the row's
// scores read from global memory) and the fused decode indexer (scores computed by the
// same CTAs and held in shared memory until the selection).
//
// Sources: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
// section 2.3 (the selector keeps the k best-scoring compressed entries) and section 4
// (k = 512 / 1024); "Follow the white rabbit: DeepSeek V4's architecture in 3D", indexer
// paragraph (top 1,024 entries at maximum context).  Ties go to the lowest index; the
// output is in ascending index order.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

namespace csa {
namespace {

struct TopkParams {
  const float* scores;
  int E_stride, k, m, cache_cap, B, E_max;
  const int32_t* q_pos;
  const int32_t* q_seq;
  const int32_t* n_entries;
  int32_t* idx;
  int32_t* cnt;
};

// order-preserving map of a float to uint32 (+0 and -0 map to the same key)
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = (f == 0.f) ? 0u : __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// block-wide exclusive scan of one value per thread; returns the exclusive prefix, total in *tot
template <int THREADS>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_buf, uint32_t* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_buf[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = lane < THREADS / 32 ? warp_buf[lane] : 0u;
    uint32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < THREADS / 32) warp_buf[lane] = wi - wv;
    if (lane == 31) *tot = wi;
  }
  __syncthreads();
  const uint32_t r = warp_buf[warp] + inc - v;
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------- register top-k
// inverse of order_key (the key of -0 maps back to +0, which compares equal)
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// A word of the shared memory of cluster CTA r (the same object in every CTA).  With
// C = 1 there is no cluster and the word is this CTA's own.
template <int C>
__device__ __forceinline__ uint32_t cta_word(const uint32_t* p, int r) {
  if constexpr (C > 1) {
    return dsmem_ld(dsmem_map(p, static_cast<uint32_t>(r)));
  } else {
    (void)r;
    return *reinterpret_cast<const volatile uint32_t*>(p);
  }
}
// N consecutive words (N = 1, 2 or a multiple of 4; the address aligned to 4 N bytes up to 16)
template <int C, int N>
__device__ __forceinline__ void cta_words(const uint32_t* p, int r, uint32_t* x) {
  if constexpr (C == 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = reinterpret_cast<const volatile uint32_t*>(p)[i];
  } else {
    const uint32_t a = dsmem_map(p, static_cast<uint32_t>(r));
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int q = 0; q < N / 4; ++q) {
        const uint4 v = dsmem_ld4(a + 16 * q);
        x[4 * q] = v.x;
        x[4 * q + 1] = v.y;
        x[4 * q + 2] = v.z;
        x[4 * q + 3] = v.w;
      }
    } else if constexpr (N == 2) {
      const uint2 v = dsmem_ld2(a);
      x[0] = v.x;
      x[1] = v.y;
    } else {
      static_assert(N == 1, "1, 2 or a multiple of 4 words");
      x[0] = dsmem_ld(a);
    }
  }
}

// barrier over every thread of the cluster (C = 1: of the CTA)
template <int C>
__device__ __forceinline__ void cta_group_sync() {
  if constexpr (C > 1) {
    cluster_sync_all();
  } else {
    __syncthreads();
  }
}

// Counts of a histogram kept per CTA (two 16-bit bins per word, buffer `h` in each of
// the C CTAs) are summed over the cluster; returns, in *s_bin and *s_above, the bin b
// with  #(bins above b) < need <= #(bins >= b).  Thread t sums the NB / THREADS bins
// [NB - (t + 1) NB / THREADS, NB - t NB / THREADS), so the scan over threads runs from
// the top bin down.
template <int C, int THREADS, int NB>
__device__ void cluster_select_bin(const uint32_t* h, uint32_t need, uint32_t* s_bin, uint32_t* s_above,
                                   uint32_t* warp_buf, uint32_t* s_tot) {
  constexpr int PER = NB / THREADS;
  static_assert(PER >= 1 && NB % THREADS == 0, "whole bins per thread");
  const int lo_bin = NB - PER * (static_cast<int>(threadIdx.x) + 1);
  constexpr int NW = PER >= 2 ? PER / 2 : 1;  // words holding this thread's bins
  uint32_t x[C][NW];
#pragma unroll
  for (int r = 0; r < C; ++r) cta_words<C, NW>(h + (lo_bin >> 1), r, x[r]);  // all in flight at once
  uint32_t c[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) c[i] = 0;
#pragma unroll
  for (int r = 0; r < C; ++r) {
    if constexpr (PER >= 2) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        c[2 * w] += x[r][w] & 0xFFFFu;
        c[2 * w + 1] += x[r][w] >> 16;
      }
    } else {
      c[0] += (x[r][0] >> ((lo_bin & 1) << 4)) & 0xFFFFu;
    }
  }
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) local += c[i];
  const uint32_t pre = block_excl_scan<THREADS>(local, warp_buf, s_tot);
  if (pre < need && need <= pre + local) {
    uint32_t acc = pre;
    bool found = false;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (!found && acc + c[i] >= need) {
        *s_bin = static_cast<uint32_t>(lo_bin + i);
        *s_above = acc;
        found = true;
      }
      acc += c[i];
    }
  }
  __syncthreads();
}

// The same search for large clusters (C >= 8) as a reduce-scatter: CTA r owns the bins
// [r NB / C, (r + 1) NB / C), sums only those over the cluster into s_own (one 32-bit count
// per bin) and publishes their total in *s_owntot; after one cluster barrier every CTA
// finds the owner of the need-th largest key from the C totals (ranked from the top bin,
// which CTA C - 1 owns) and scans that owner's bins.  A CTA reads 2 NB / C + NB / C words
// of distributed shared memory instead of C NB / 2 (for C = 16 and NB = 4096: 1.5 KB per
// thread block instead of 128 KB), at the price of that barrier.  The caller has
// synchronised the cluster after the histograms were complete; s_own and *s_owntot are
// rewritten only after the next such barrier.
template <int C, int THREADS, int NB>
__device__ void cluster_select_bin_rs(const uint32_t* h, uint32_t need, int rank, uint32_t* s_bin, uint32_t* s_above,
                                      uint32_t* warp_buf, uint32_t* s_tot, uint32_t* s_own, uint32_t* s_owntot,
                                      uint32_t* s_sel) {
  constexpr int OWN = NB / C;   // bins a CTA owns
  constexpr int OWNW = OWN / 2;  // their words
  static_assert(C >= 2 && C <= 32 && NB % (2 * C) == 0 && OWNW <= THREADS, "owned words: one per thread at most");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t mine = 0;
  if (static_cast<int>(threadIdx.x) < OWNW) {
    const uint32_t* w = h + rank * OWNW + threadIdx.x;
    uint32_t x[C];
#pragma unroll
    for (int r = 0; r < C; ++r) x[r] = cta_word<C>(w, r);  // all in flight at once
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int r = 0; r < C; ++r) {
      lo += x[r] & 0xFFFFu;
      hi += x[r] >> 16;
    }
    s_own[2 * threadIdx.x] = lo;
    s_own[2 * threadIdx.x + 1] = hi;
    mine = lo + hi;
  }
  block_excl_scan<THREADS>(mine, warp_buf, s_tot);
  if (threadIdx.x == 0) *s_owntot = *s_tot;
  cta_group_sync<C>();  // every CTA's owned sums and total are published
  if (warp == 0) {
    const uint32_t t = lane < C ? cta_word<C>(s_owntot, lane) : 0u;
    uint32_t suf = t;  // inclusive suffix sum over lanes (CTA C - 1 owns the top bins)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += y;
    }
    const uint32_t above_r = suf - t;
    const uint32_t who = __ballot_sync(0xffffffffu, lane < C && above_r < need && need <= suf);
    const int owner = who ? __ffs(who) - 1 : 0;
    if (lane == owner) {
      s_sel[0] = static_cast<uint32_t>(owner);
      s_sel[1] = above_r;
    }
  }
  __syncthreads();
  const int owner = static_cast<int>(s_sel[0]);
  const uint32_t base = s_sel[1];
  // the owner's bins from the top: thread t takes [OWN - (t + 1) PER, OWN - t PER)
  constexpr int PER = (OWN + THREADS - 1) / THREADS;
  const int lo_bin = OWN - PER * (static_cast<int>(threadIdx.x) + 1);
  uint32_t c[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) c[i] = lo_bin + i >= 0 ? cta_word<C>(s_own + lo_bin + i, owner) : 0u;
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) local += c[i];
  const uint32_t pre = base + block_excl_scan<THREADS>(local, warp_buf, s_tot);
  if (pre < need && need <= pre + local) {
    uint32_t acc = pre;
    bool found = false;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (!found && acc + c[i] >= need) {
        *s_bin = static_cast<uint32_t>(owner * OWN + lo_bin + i);
        *s_above = acc;
        found = true;
      }
      acc += c[i];
    }
  }
  __syncthreads();
}

// add one key to bin b of a histogram of 16-bit counts, two per word
__device__ __forceinline__ void hist16_add(uint32_t* h, uint32_t b) { atomicAdd(&h[b >> 1], 1u << ((b & 1u) << 4)); }

template <int EPT>
using TopkMask = typename std::conditional<(EPT > 32), unsigned long long, uint32_t>::type;

// Exact top-k of one query row held in registers by a cluster of C CTAs (C = 1: one CTA).
// CTA r of the cluster holds entries [r S, (r + 1) S), S = THREADS EPT; within it warp w
// owns the contiguous chunk [32 EPT w, 32 EPT (w + 1)) and its lane l holds entries
// 32 EPT w + 32 i + l for i < EPT (each load instruction of a warp reads 128 contiguous
// bytes).  Steps:
//   range     min / max of the row: each CTA's pair, combined over the cluster
//   bins      4096 linear bins over the range, b(x) = min(round(x inv - lo inv), 4095),
//             monotone in x; each CTA counts its slice and every CTA sums the cluster's
//             counts (distributed shared memory) to find the bin holding the k-th largest
//   threshold that bin's members give the exact k-th key: one warp ranks up to 32 members
//             of the cluster directly; more go through three MSB digit passes (12, 10, 10
//             bits) restricted to the members, each summed over the cluster the same way
//   output    per i, two ballots give the masks of the 32 contiguous entries
//             [32 EPT w + 32 i, +32), which lane i mod 32 keeps; a scan over lanes and
//             warps, plus the kept counts of the CTAs before this one, gives each kept
//             entry (above the threshold, or among the lowest-index ties) its slot
// Histogram buffers alternate (0: bins, 1: digit 0, 0: digit 1, 1: digit 2) so that a
// buffer is rewritten only after a cluster barrier that every CTA reaches after reading it.
// The row's entries [rank S, (rank + 1) S) are in v (entry of v[i] at thread (warp w, lane
// l): rank S + 32 EPT w + 32 i + l), `valid` marks the visible ones (bit i for v[i]); the
// row has more than p.k visible entries.  Writes p.idx[row, :] and p.cnt[row].  Every
// thread of every CTA of the cluster calls it.
template <int C, int THREADS, int EPT>
__device__ __forceinline__ void topk_regs_row(const TopkParams& p, int row, int rank, const float (&v)[EPT],
                                              TopkMask<EPT> valid) {
  static_assert(EPT == 8 || EPT == 16 || EPT == 32 || EPT == 64, "EPT: 8, 16, 32 or 64 entries per thread");
  static_assert(C == 1 || C == 2 || C == 4 || C == 8 || C == 16, "cluster sizes: 1 to 8 (portable) or 16");
  constexpr int kRedLanes = C > 8 ? 16 : 8;  // lanes of warp 0 holding one CTA's value each
  static_assert(THREADS * EPT <= 32768, "a CTA's count in one bin fits 16 bits");
  using Mask = TopkMask<EPT>;
  constexpr Mask kOne = 1;
  constexpr int kBins = 4096;
  constexpr int kWarps = THREADS / 32;
  constexpr int kHalves = EPT > 32 ? 2 : 1;  // 32-entry groups a lane keeps in the output step
  constexpr int kSlice = THREADS * EPT;      // entries per CTA
  static_assert(kBins % THREADS == 0 && 1024 % THREADS == 0, "bin scans assume whole bins per thread");
  __shared__ __align__(16) uint32_t hist[2][kBins / 2];  // this CTA's counts, two 16-bit bins per word
  __shared__ uint32_t warp_buf[32], s_tot, s_bin, s_above, s_ncand, s_zero, s_total;
  __shared__ float s_red[2][32];
  __shared__ __align__(8) uint32_t s_range[2];  // this CTA's min / max (float bits)
  __shared__ float s_grange[2];            // the row's
  __shared__ uint32_t s_cand[32];          // this CTA's first 32 member keys
  __shared__ uint32_t s_thr[2];
  // reduce-scatter search (C >= 8): this CTA's owned bin sums, their total, the owner found
  __shared__ uint32_t s_own[C >= 8 ? kBins / C : 1], s_owntot, s_sel[2];
  __shared__ __align__(8) uint32_t s_cnt[2];  // this CTA's kept counts: above the threshold, equal to it
  __shared__ uint32_t s_cbase[2];          // the same summed over the CTAs before this one
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wbase = rank * kSlice + 32 * EPT * warp;
  int32_t* out = p.idx + static_cast<size_t>(row) * p.k;
  const int tslot = (row < 2 && rank == 0 && threadIdx.x == 0) ? 2 + row : -1;
  (void)tslot;  // phase stamps only in timing builds
  for (int b = threadIdx.x; b < kBins / 2; b += THREADS) hist[0][b] = 0;
  if (threadIdx.x == 0) {
    s_ncand = 0;
    s_zero = 0;
  }
  CSA_T(tslot, 5);

  // Per-slot passes come in two forms: a fully visible warp chunk (the common case, no
  // per-slot validity test) and a partial one.
  const bool full = valid == ~Mask(0);  // warp-uniform
  auto slots = [&](auto body) {
    if (full) {
#pragma unroll
      for (int i = 0; i < EPT; ++i) body(i, true);
    } else {
#pragma unroll
      for (int i = 0; i < EPT; ++i) body(i, (valid >> i & kOne) != 0);
    }
  };

  // ---- range of the row
  float lo = INFINITY, hi = -INFINITY;
  slots([&](int i, bool ok) {
    if (ok) {
      lo = fminf(lo, v[i]);
      hi = fmaxf(hi, v[i]);
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    s_red[0][warp] = lo;
    s_red[1][warp] = hi;
  }
  __syncthreads();
  if (warp == 0) {
    lo = lane < kWarps ? s_red[0][lane] : INFINITY;
    hi = lane < kWarps ? s_red[1][lane] : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      s_range[0] = __float_as_uint(lo);
      s_range[1] = __float_as_uint(hi);
    }
  }
  CSA_T(tslot, 6);
  cta_group_sync<C>();  // every CTA's range is published
  CSA_T(tslot, 7);
  if (warp == 0) {
    uint32_t rg[2] = {__float_as_uint(INFINITY), __float_as_uint(-INFINITY)};
    if (lane < C) cta_words<C, 2>(s_range, lane, rg);
    lo = __uint_as_float(rg[0]);
    hi = __uint_as_float(rg[1]);
#pragma unroll
    for (int o = kRedLanes / 2; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      s_grange[0] = lo;
      s_grange[1] = hi;
    }
  }
  __syncthreads();
  lo = s_grange[0];
  hi = s_grange[1];
  const float span = hi - lo;
  const float inv = (span > 0.f && span < INFINITY) ? static_cast<float>(kBins - 1) / span : 0.f;
  const float nlo = inv > 0.f ? -lo * inv : 0.f;
  // Bin of x: round(clamp(x inv - lo inv, 0, 4095)), monotone non-decreasing in x (an fma of
  // an increasing affine map, then a clamp and a rounding); NaN -> 0.  Adding 1.5 * 2^23
  // leaves the rounded integer in the low mantissa bits (no float-to-int conversion).
  auto bin_of = [&](float x, float c) -> uint32_t {
    const float f = fminf(fmaxf(fmaf(x, inv, c), 0.f), static_cast<float>(kBins - 1));
    return __float_as_uint(f + 12582912.0f) - 0x4B400000u;
  };
  CSA_T(tslot, 1);

  // ---- histogram and the bin holding the k-th largest
  slots([&](int i, bool ok) {
    if (ok) hist16_add(hist[0], bin_of(v[i], nlo));
  });
  CSA_T(tslot, 8);
  cta_group_sync<C>();  // every CTA's counts are complete
  CSA_T(tslot, 9);
  if constexpr (C >= 8)
    cluster_select_bin_rs<C, THREADS, kBins>(hist[0], static_cast<uint32_t>(p.k), rank, &s_bin, &s_above, warp_buf,
                                             &s_tot, s_own, &s_owntot, s_sel);
  else
    cluster_select_bin<C, THREADS, kBins>(hist[0], static_cast<uint32_t>(p.k), &s_bin, &s_above, warp_buf, &s_tot);
  const uint32_t b1 = s_bin;
  const uint32_t above1 = s_above;
  CSA_T(tslot, 2);

  // ---- members of that bin (every key above them lies in a higher bin).  The offset is
  // re-read from shared memory (it is zero plus nlo) so that the compiler recomputes the
  // bins here instead of keeping EPT of them live across the scan.
  Mask mem = 0;
  {
    const float c = nlo + __uint_as_float(*reinterpret_cast<volatile const uint32_t*>(&s_zero));
    slots([&](int i, bool ok) {
      if (ok && bin_of(v[i], c) == b1) mem |= kOne << i;
    });
  }
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    if (mem >> i & kOne) {
      const uint32_t slot = atomicAdd(&s_ncand, 1u);
      if (slot < 32u) s_cand[slot] = order_key(v[i]);
    }
  }
  CSA_T(tslot, 10);
  cta_group_sync<C>();  // every CTA's member count and first member keys are published
  CSA_T(tslot, 11);
  const uint32_t need = static_cast<uint32_t>(p.k) - above1;  // 1 <= need <= members
  if (warp == 0) {
    // members per CTA, their prefix in CTA order, and the cluster total
    // one round of loads: lane l reads the count of CTA l and word l of every CTA's list
    uint32_t cand[C];
#pragma unroll
    for (int r = 0; r < C; ++r) cand[r] = cta_word<C>(&s_cand[lane], r);
    const uint32_t nc = lane < C ? cta_word<C>(&s_ncand, lane) : 0u;
    uint32_t incl = nc;
#pragma unroll
    for (int o = 1; o < kRedLanes; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, kRedLanes - 1);
    if (total <= 32u) {
      // lane j < total fetches the j-th member key (CTAs in order), then the warp ranks them
      uint32_t key = 0;
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t hi_r = __shfl_sync(0xffffffffu, incl, r);
        const uint32_t lo_r = hi_r - __shfl_sync(0xffffffffu, nc, r);
        const uint32_t kr = __shfl_sync(0xffffffffu, cand[r], (static_cast<uint32_t>(lane) - lo_r) & 31u);
        if (static_cast<uint32_t>(lane) >= lo_r && static_cast<uint32_t>(lane) < hi_r) key = kr;
      }
      uint32_t g = 0, ge = 0;
      for (int j = 0; j < static_cast<int>(total); ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
        g += kj > key ? 1u : 0u;
        ge += kj >= key ? 1u : 0u;
      }
      const bool is_thr = lane < static_cast<int>(total) && g < need && need <= ge;
      const uint32_t who = __ballot_sync(0xffffffffu, is_thr);
      if (who != 0u && lane == __ffs(who) - 1) {
        s_thr[0] = key;
        s_thr[1] = g;
      }
    }
    if (lane == 0) s_total = total;
  }
  __syncthreads();
  uint32_t thr, above_c;
  if (s_total <= 32u) {  // the same decision in every CTA of the cluster
    thr = s_thr[0];
    above_c = s_thr[1];
  } else {
    // MSB digit passes over the members' keys; each pass re-derives the keys from a zero
    // re-read from shared memory rather than keeping EPT of them live
    uint32_t prefix = 0, above = 0;
    auto digit_pass = [&](auto nb_tag, uint32_t* h, int shift, bool first) {
      constexpr int NB = decltype(nb_tag)::value;
      constexpr int kWidth = NB == 4096 ? 12 : 10;
      for (int b = threadIdx.x; b < NB / 2; b += THREADS) h[b] = 0;
      __syncthreads();
      const float z = __uint_as_float(*reinterpret_cast<volatile const uint32_t*>(&s_zero));
#pragma unroll
      for (int i = 0; i < EPT; ++i) {
        if (mem >> i & kOne) {
          const uint32_t key = order_key(v[i] + z);  // x + 0 keeps the key (-0 and +0 share one)
          if (first || (key >> (shift + kWidth)) == prefix) hist16_add(h, (key >> shift) & static_cast<uint32_t>(NB - 1));
        }
      }
      cta_group_sync<C>();
      if constexpr (C >= 8)
        cluster_select_bin_rs<C, THREADS, NB>(h, need - above, rank, &s_bin, &s_above, warp_buf, &s_tot, s_own,
                                              &s_owntot, s_sel);
      else
        cluster_select_bin<C, THREADS, NB>(h, need - above, &s_bin, &s_above, warp_buf, &s_tot);
      prefix = (prefix << kWidth) | s_bin;
      above += s_above;
      __syncthreads();
    };
    digit_pass(std::integral_constant<int, 4096>{}, hist[1], 20, true);
    digit_pass(std::integral_constant<int, 1024>{}, hist[0], 10, false);
    digit_pass(std::integral_constant<int, 1024>{}, hist[1], 0, false);
    thr = prefix;
    above_c = above;
  }
  const uint32_t ties = static_cast<uint32_t>(p.k) - (above1 + above_c);  // lowest-index thr keys to keep
  const float thr_f = key_float(thr);
  CSA_T(tslot, 3);

  // ---- ordered output: slot of an entry = #above before it + min(#equal before it, ties)
  uint32_t mg[kHalves], me[kHalves];
#pragma unroll
  for (int h = 0; h < kHalves; ++h) mg[h] = me[h] = 0;
  slots([&](int i, bool ok) {
    const uint32_t bg = __ballot_sync(0xffffffffu, ok && v[i] > thr_f);
    const uint32_t be = __ballot_sync(0xffffffffu, ok && v[i] == thr_f);
    if (lane == (i & 31)) {
      mg[i >> 5] = bg;
      me[i >> 5] = be;
    }
  });
  // kept counts in order (half 0 lanes 0..31, then half 1), both <= 32768: 16-bit halves
  uint32_t incl[kHalves], cnt[kHalves];
  uint32_t wsum = 0;
#pragma unroll
  for (int h = 0; h < kHalves; ++h) {
    cnt[h] = (static_cast<uint32_t>(__popc(mg[h])) << 16) | static_cast<uint32_t>(__popc(me[h]));
    uint32_t x = cnt[h];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    incl[h] = x + wsum;
    wsum += __shfl_sync(0xffffffffu, x, 31);
  }
  CSA_T(tslot, 12);
  const uint32_t wpre = __shfl_sync(0xffffffffu, block_excl_scan<THREADS>(lane == 0 ? wsum : 0u, warp_buf, &s_tot), 0);
  CSA_T(tslot, 13);
  uint32_t base_g = 0, base_q = 0;
  if constexpr (C > 1) {
    if (threadIdx.x == 0) {
      s_cnt[0] = s_tot >> 16;
      s_cnt[1] = s_tot & 0xFFFFu;
    }
    cta_group_sync<C>();  // every CTA's kept counts are published
    if (warp == 0) {
      uint32_t gq[2] = {0u, 0u};
      if (lane < rank) cta_words<C, 2>(s_cnt, lane, gq);
      uint32_t g = gq[0], q = gq[1];
#pragma unroll
      for (int o = kRedLanes / 2; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        q += __shfl_xor_sync(0xffffffffu, q, o);
      }
      if (lane == 0) {
        s_cbase[0] = g;
        s_cbase[1] = q;
      }
    }
    cluster_arrive();  // this CTA reads no other CTA's shared memory after this point
    __syncthreads();
    CSA_T(tslot, 14);
    base_g = s_cbase[0];
    base_q = s_cbase[1];
  }
#pragma unroll
  for (int h = 0; h < kHalves; ++h) {
    const uint32_t pre = wpre + incl[h] - cnt[h];
    const uint32_t g = base_g + (pre >> 16), q = base_q + (pre & 0xFFFFu);
    const int gbase = wbase + 32 * (32 * h + lane);  // first entry of the kept group
    for (uint32_t sel = mg[h] | me[h]; sel != 0u; sel &= sel - 1u) {
      const int j = __ffs(sel) - 1;
      const uint32_t below = (1u << j) - 1u;
      const uint32_t gb = g + __popc(mg[h] & below), qb = q + __popc(me[h] & below);
      uint32_t at = 0xFFFFFFFFu;
      if (mg[h] >> j & 1u) at = gb + min(qb, ties);
      else if (qb < ties) at = gb + qb;
      if (at < static_cast<uint32_t>(p.k)) out[at] = gbase + j;  // NaN scores can break the count
    }
  }
  if (rank == 0 && threadIdx.x == 0) p.cnt[row] = p.k;
  CSA_T(tslot, 15);
  if constexpr (C > 1) cluster_wait();  // no CTA leaves while another may still read its shared memory
  CSA_T(tslot, 4);
}

}  // namespace
}  // namespace csa
