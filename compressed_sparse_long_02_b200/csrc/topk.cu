// topk.cu -- exact top-k selection of indexer scores, ties to the lowest index, output
// in ascending index order (padded with -1 when fewer than k entries are visible).
//
// Sources: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
// §2.3 (the selector keeps the k best-scoring compressed entries) and §4 (k = 512 /
// 1024); "Follow the white rabbit: DeepSeek V4's architecture in 3D", indexer paragraph
// (top 1,024 entries at maximum context).
//
// Two kernels compute the same result:
//   topk_kernel          one CTA per query row (many rows: prefill)
//   topk_cluster_kernel  one thread-block cluster of C CTAs per row (few long rows:
//                        decode); each CTA owns a contiguous slice of the row and the
//                        CTAs exchange histograms and counts through distributed
//                        shared memory.
// Both bin the row's scores linearly over [min, max] (monotone in the score), find the
// bin holding the k-th largest, resolve the exact k-th key by an MSB radix select over
// that bin's members (order-preserving float -> uint key), and write every score above
// the threshold plus the lowest-index ties with an order-preserving ballot compaction.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
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

__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t peers = __match_any_sync(0xffffffffu, active ? bin : 0xFFFFFFFFu);
  if (active && (threadIdx.x & 31) == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
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

// Find bin b with  #(bins above b) < need <= #(bins >= b).  Bins are scanned from the top.
template <int THREADS>
__device__ void select_bin(const uint32_t* hist, int nbins, uint32_t need, uint32_t* s_bin, uint32_t* s_above,
                           uint32_t* warp_buf, uint32_t* tot) {
  const int per = nbins / THREADS;
  const int hi = nbins - per * static_cast<int>(threadIdx.x);  // bins [hi-per, hi)
  uint32_t local = 0;
  for (int i = 1; i <= per; ++i) local += hist[hi - i];
  const uint32_t pre = block_excl_scan<THREADS>(local, warp_buf, tot);
  if (pre < need && need <= pre + local) {
    uint32_t acc = pre;
    for (int i = 1; i <= per; ++i) {
      const uint32_t c = hist[hi - i];
      if (acc + c >= need) {
        *s_bin = static_cast<uint32_t>(hi - i);
        *s_above = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// Exact selection of the `need`-th largest key among n keys: three MSB digit passes
// (12, 10, 10 bits).  Returns the threshold key and the number of keys above it.
template <int THREADS, typename KeyFn>
__device__ void radix_select(KeyFn key_of, int n, uint32_t need, uint32_t* hist, uint32_t* warp_buf,
                             uint32_t* s_tot, uint32_t* s_bin, uint32_t* s_above, uint32_t& thr_out,
                             uint32_t& above_out) {
  uint32_t prefix = 0, above = 0;
  const int shifts[3] = {20, 10, 0};
  const int widths[3] = {12, 10, 10};
#pragma unroll 1
  for (int d = 0; d < 3; ++d) {
    const int nb = 1 << widths[d];
    for (int i = threadIdx.x; i < nb; i += THREADS) hist[i] = 0;
    __syncthreads();
    const int hi_shift = shifts[d] + widths[d];
    for (int base = 0; base < n; base += THREADS) {
      const int j = base + threadIdx.x;
      const bool in = j < n;
      const uint32_t key = in ? key_of(j) : 0u;
      const bool act = in && (d == 0 || (key >> hi_shift) == prefix);
      warp_hist_add(hist, (key >> shifts[d]) & static_cast<uint32_t>(nb - 1), act);
    }
    __syncthreads();
    select_bin<THREADS>(hist, nb, need - above, s_bin, s_above, warp_buf, s_tot);
    prefix = (prefix << widths[d]) | *s_bin;
    above += *s_above;
    __syncthreads();
  }
  thr_out = prefix;
  above_out = above;
}

// One CTA per query row.  The row is staged in shared memory with all loads in flight;
// scores are binned linearly over [min, max] of the row (an order-preserving map that
// spreads concentrated score distributions over 4096 bins), the bin holding the k-th
// largest is resolved exactly by radix select over its members, and an ordered
// compaction writes every score above the threshold plus the lowest-index ties.  If
// the threshold bin holds more members than the candidate buffer, the radix select
// runs over the whole row instead (same result, slower).
template <int THREADS>
__global__ void __launch_bounds__(THREADS) topk_kernel(TopkParams p) {
  griddep_enter();
  extern __shared__ __align__(16) uint32_t tsm[];
  constexpr int kCandCap = 8192;
  uint32_t* hist = tsm;                 // 4096 bins
  uint32_t* cand = tsm + 4096;          // candidate keys
  uint32_t* rowbits = cand + kCandCap;  // cached score bits (cache_cap)
  __shared__ uint32_t warp_buf[32], s_tot, s_bin, s_above, s_ncand;
  __shared__ float s_red[2][32];

  const int row = blockIdx.x;
  const int seq = p.q_seq[row];
  const int nv = (seq < 0 || seq >= p.B) ? 0 : min(visible_entries(p.q_pos[row], p.m, p.n_entries[seq]), p.E_max);
  int32_t* out = p.idx + static_cast<size_t>(row) * p.k;
  if (nv <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += THREADS) out[j] = j < nv ? j : -1;
    if (threadIdx.x == 0) p.cnt[row] = nv;
    return;
  }
  const float* src = p.scores + static_cast<size_t>(row) * p.E_stride;
  const bool cached = nv <= p.cache_cap;
  const int tslot = (row < 2 && threadIdx.x == 0) ? 2 + row : -1;
  CSA_T(tslot, 0);
  if (cached) {
    const int n4 = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 ? nv / 4 : 0;
    for (int c = threadIdx.x; c < n4; c += THREADS) cp_async_16(smem_u32(rowbits + 4 * c), src + 4 * c, true);
    for (int j = 4 * n4 + threadIdx.x; j < nv; j += THREADS) rowbits[j] = __float_as_uint(__ldg(src + j));
    cp_async_wait_all();
    __syncthreads();
  }
  CSA_T(tslot, 1);
  auto val = [&](int j) -> float { return cached ? __uint_as_float(rowbits[j]) : __ldg(src + j); };
  auto key_at = [&](int j) -> uint32_t { return order_key(val(j)); };
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = THREADS / 32;

  // row range
  float lo = INFINITY, hi = -INFINITY;
  for (int j = threadIdx.x; j < nv; j += THREADS) {
    const float x = val(j);
    lo = fminf(lo, x);
    hi = fmaxf(hi, x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    s_red[0][warp] = lo;
    s_red[1][warp] = hi;
  }
  for (int i = threadIdx.x; i < 4096; i += THREADS) hist[i] = 0;
  if (threadIdx.x == 0) s_ncand = 0;
  __syncthreads();
  lo = s_red[0][0];
  hi = s_red[1][0];
  for (int w = 1; w < kWarps; ++w) {
    lo = fminf(lo, s_red[0][w]);
    hi = fmaxf(hi, s_red[1][w]);
  }
  const float span = hi - lo;
  const float inv = (span > 0.f && span < INFINITY) ? 4095.0f / span : 0.f;
  auto bin_of = [&](float x) -> uint32_t {  // monotone non-decreasing in x
    const float f = (x - lo) * inv;
    const uint32_t b = f > 0.f ? static_cast<uint32_t>(f) : 0u;
    return b > 4095u ? 4095u : b;
  };

  // linear-bin histogram and the bin holding the k-th largest score
  CSA_T(tslot, 2);
  for (int j = threadIdx.x; j < nv; j += THREADS) atomicAdd(&hist[bin_of(val(j))], 1u);
  __syncthreads();
  CSA_T(tslot, 3);
  select_bin<THREADS>(hist, 4096, static_cast<uint32_t>(p.k), &s_bin, &s_above, warp_buf, &s_tot);
  const uint32_t b1 = s_bin;
  const uint32_t above1 = s_above;
  CSA_T(tslot, 4);
  // members of that bin (keys strictly above lie in higher bins, below in lower ones)
  for (int j = threadIdx.x; j < nv; j += THREADS) {
    const float x = val(j);
    if (bin_of(x) == b1) {
      const uint32_t slot = atomicAdd(&s_ncand, 1u);
      if (slot < kCandCap) cand[slot] = order_key(x);
    }
  }
  __syncthreads();
  const int ncand = static_cast<int>(s_ncand);
  CSA_T(tslot, 5);
  if (tslot >= 0) CSA_T(tslot, 40 + (ncand > 8192 ? 1 : 0));
  uint32_t thr, n_above;
  if (ncand <= kCandCap) {
    uint32_t above_c;
    radix_select<THREADS>([&](int i) { return cand[i]; }, ncand, static_cast<uint32_t>(p.k) - above1, hist, warp_buf,
                          &s_tot, &s_bin, &s_above, thr, above_c);
    n_above = above1 + above_c;
  } else {
    radix_select<THREADS>(key_at, nv, static_cast<uint32_t>(p.k), hist, warp_buf, &s_tot, &s_bin, &s_above, thr,
                          n_above);
  }
  const uint32_t ties = static_cast<uint32_t>(p.k) - n_above;  // lowest-index keys equal to thr to keep
  CSA_T(tslot, 6);

  // ordered output: each warp owns a contiguous chunk; lanes stride through it so that
  // ballots preserve index order
  const int chunk = ((nv + kWarps - 1) / kWarps + 31) & ~31;
  const int c_lo = warp * chunk, c_hi = min(nv, c_lo + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = c_lo; base < c_hi; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < c_hi ? key_at(j) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, j < c_hi && key > thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, j < c_hi && key == thr));
  }
  const uint32_t gt_pre = block_excl_scan<THREADS>(lane == 0 ? n_gt : 0u, warp_buf, &s_tot);
  const uint32_t eq_pre = block_excl_scan<THREADS>(lane == 0 ? n_eq : 0u, warp_buf, &s_tot);
  uint32_t gt_base = __shfl_sync(0xffffffffu, gt_pre, 0);
  uint32_t eq_base = __shfl_sync(0xffffffffu, eq_pre, 0);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = c_lo; base < c_hi; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < c_hi ? key_at(j) : 0u;
    const uint32_t bgt = __ballot_sync(0xffffffffu, j < c_hi && key > thr);
    const uint32_t beq = __ballot_sync(0xffffffffu, j < c_hi && key == thr);
    const uint32_t eq_before = eq_base + __popc(beq & lt_mask);
    const bool take = (bgt >> lane & 1u) || ((beq >> lane & 1u) && eq_before < ties);
    const uint32_t at = gt_base + __popc(bgt & lt_mask) + min(eq_before, ties);
    if (take && at < static_cast<uint32_t>(p.k)) out[at] = j;  // NaN scores can break the count
    gt_base += __popc(bgt);
    eq_base += __popc(beq);
  }
  if (threadIdx.x == 0) p.cnt[row] = p.k;
  CSA_T(tslot, 7);
}


// ---------------------------------------------------------------------- register top-k
// inverse of order_key (the key of -0 maps back to +0, which compares equal)
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// One CTA per query row with the whole row in registers.  Warp w owns the contiguous
// chunk [32 EPT w, 32 EPT (w + 1)); its lane l holds entries 32 EPT w + 32 i + l for
// i < EPT (each load instruction of a warp reads 128 contiguous bytes).  Steps:
//   range     min / max of the row
//   bins      4096 linear bins over the range, b(x) = min(trunc(x inv - lo inv), 4095),
//             monotone in x; the bin holding the k-th largest score
//   threshold that bin's members (a bit mask per thread) give the exact k-th key: one
//             warp ranks at most 32 members directly, more go through three MSB digit
//             passes restricted to the members
//   output    per i, two ballots give the masks of the 32 contiguous entries
//             [32 EPT w + 32 i, +32), which lane i mod 32 keeps; a scan over lanes and
//             warps of the kept counts gives each entry its slot in index order
template <int THREADS, int EPT>
__global__ void __launch_bounds__(THREADS) topk_reg_kernel(TopkParams p) {
  static_assert(EPT == 16 || EPT == 32 || EPT == 64, "EPT: 16, 32 or 64 entries per thread");
  using Mask = typename std::conditional<(EPT > 32), unsigned long long, uint32_t>::type;
  constexpr Mask kOne = 1;
  constexpr int kBins = 4096;
  constexpr int kWarps = THREADS / 32;
  constexpr int kHalves = EPT > 32 ? 2 : 1;  // 32-entry groups a lane keeps in the output step
  static_assert(kBins % THREADS == 0 && 1024 % THREADS == 0, "bin scans assume whole bins per thread");
  griddep_enter();
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_buf[32], s_tot, s_bin, s_above, s_ncand, s_zero;
  __shared__ float s_red[2][32];
  __shared__ float s_range[2];
  __shared__ uint32_t s_cand[32];
  __shared__ uint32_t s_thr[2];

  const int row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seq = p.q_seq[row];
  const int nv = (seq < 0 || seq >= p.B) ? 0 : min(visible_entries(p.q_pos[row], p.m, p.n_entries[seq]), p.E_max);
  int32_t* out = p.idx + static_cast<size_t>(row) * p.k;
  if (nv <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += THREADS) out[j] = j < nv ? j : -1;
    if (threadIdx.x == 0) p.cnt[row] = nv;
    return;
  }
  const int tslot = (row < 2 && threadIdx.x == 0) ? 2 + row : -1;
  CSA_T(tslot, 0);

  // ---- the row into registers
  const int wbase = 32 * EPT * warp;
  const int e0 = wbase + lane;  // entry of v[i] is e0 + 32 i
  const float* src = p.scores + static_cast<size_t>(row) * p.E_stride + e0;
  float v[EPT];
  Mask valid;
  if (wbase + 32 * EPT <= nv) {  // warp-uniform: the whole chunk is visible
#pragma unroll
    for (int i = 0; i < EPT; ++i) v[i] = __ldg(src + 32 * i);
    valid = ~Mask(0);
  } else {
    valid = 0;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const bool ok = e0 + 32 * i < nv;
      v[i] = ok ? __ldg(src + 32 * i) : 0.f;
      valid |= (ok ? kOne : Mask(0)) << i;
    }
  }
  for (int b = threadIdx.x; b < kBins; b += THREADS) hist[b] = 0;
  if (threadIdx.x == 0) {
    s_ncand = 0;
    s_zero = 0;
  }

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
      s_range[0] = lo;
      s_range[1] = hi;
    }
  }
  __syncthreads();
  lo = s_range[0];
  hi = s_range[1];
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
    if (ok) atomicAdd(&hist[bin_of(v[i], nlo)], 1u);
  });
  __syncthreads();
  select_bin<THREADS>(hist, kBins, static_cast<uint32_t>(p.k), &s_bin, &s_above, warp_buf, &s_tot);
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
  __syncthreads();
  const uint32_t ncand = s_ncand;
  const uint32_t need = static_cast<uint32_t>(p.k) - above1;  // 1 <= need <= ncand
  uint32_t thr, above_c;
  if (ncand <= 32u) {
    // one warp ranks the members directly
    if (warp == 0) {
      const uint32_t key = lane < static_cast<int>(ncand) ? s_cand[lane] : 0u;
      uint32_t g = 0, ge = 0;
      for (int j = 0; j < static_cast<int>(ncand); ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
        g += kj > key ? 1u : 0u;
        ge += kj >= key ? 1u : 0u;
      }
      const bool is_thr = lane < static_cast<int>(ncand) && g < need && need <= ge;
      const uint32_t who = __ballot_sync(0xffffffffu, is_thr);
      if (who != 0u && lane == __ffs(who) - 1) {
        s_thr[0] = key;
        s_thr[1] = g;
      }
    }
    __syncthreads();
    thr = s_thr[0];
    above_c = s_thr[1];
  } else {
    // three MSB digit passes (12, 10, 10 bits) over the members' keys; each pass re-derives
    // the keys from a zero re-read from shared memory rather than keeping EPT of them live
    uint32_t prefix = 0, above = 0;
    const int shifts[3] = {20, 10, 0};
    const int widths[3] = {12, 10, 10};
#pragma unroll 1
    for (int d = 0; d < 3; ++d) {
      const int nb = 1 << widths[d];
      for (int b = threadIdx.x; b < nb; b += THREADS) hist[b] = 0;
      __syncthreads();
      const int hi_shift = shifts[d] + widths[d];
      const float z = __uint_as_float(*reinterpret_cast<volatile const uint32_t*>(&s_zero));
#pragma unroll
      for (int i = 0; i < EPT; ++i) {
        if (mem >> i & kOne) {
          const uint32_t key = order_key(v[i] + z);  // x + 0 keeps the key (-0 and +0 share one)
          if (d == 0 || (key >> hi_shift) == prefix)
            atomicAdd(&hist[(key >> shifts[d]) & static_cast<uint32_t>(nb - 1)], 1u);
        }
      }
      __syncthreads();
      select_bin<THREADS>(hist, nb, need - above, &s_bin, &s_above, warp_buf, &s_tot);
      prefix = (prefix << widths[d]) | s_bin;
      above += s_above;
      __syncthreads();
    }
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
  const uint32_t wpre = __shfl_sync(0xffffffffu, block_excl_scan<THREADS>(lane == 0 ? wsum : 0u, warp_buf, &s_tot), 0);
#pragma unroll
  for (int h = 0; h < kHalves; ++h) {
    const uint32_t pre = wpre + incl[h] - cnt[h];
    const uint32_t g = pre >> 16, q = pre & 0xFFFFu;
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
  if (threadIdx.x == 0) p.cnt[row] = p.k;
  CSA_T(tslot, 4);
}

int g_topk_smem[2][64];

}  // namespace

cudaError_t launch_topk_select(const IndexArgs& a, cudaStream_t s) {
  TopkParams t{};
  t.scores = a.scores_ws;
  t.E_stride = a.E_stride;
  t.k = a.k;
  t.m = a.m;
  t.B = a.B;
  t.E_max = a.E_max;
  t.q_pos = a.q_pos;
  t.q_seq = a.q_seq;
  t.n_entries = a.n_entries;
  t.idx = a.idx_out;
  t.cnt = a.cnt_out;
  cudaError_t e;
  // rows that fit in registers: up to 32 entries per thread
  if (a.E_max <= 2048) {
    e = launch_pdl(topk_reg_kernel<128, 16>, dim3(a.Nq), dim3(128), 0, s, t);
  } else if (a.E_max <= 8192) {
    e = launch_pdl(topk_reg_kernel<256, 32>, dim3(a.Nq), dim3(256), 0, s, t);
  } else if (a.E_max <= 32768) {
    e = launch_pdl(topk_reg_kernel<1024, 32>, dim3(a.Nq), dim3(1024), 0, s, t);
  } else {
    // longer rows: staged in shared memory (read from global beyond its capacity)
    const int max_dyn = 227 * 1024 - 1024;  // room for the kernel's static shared memory
    const int cache_cap = std::min(a.E_max, (max_dyn - (4096 + 8192) * 4) / 4);
    t.cache_cap = cache_cap;
    const size_t tsmem = (4096 + 8192 + static_cast<size_t>(cache_cap)) * 4;
    e = set_dyn_smem(reinterpret_cast<const void*>(topk_kernel<1024>), tsmem, g_topk_smem[1]);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_kernel<1024>, dim3(a.Nq), dim3(1024), tsmem, s, t);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa
