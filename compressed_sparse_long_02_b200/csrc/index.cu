// index_topk.cu -- lightning indexer (block-scaled FP4 tcgen05 contraction) and
// exact radix top-k.
//
// Sources: "DeepSeek-V4: Million-Token Context", CSA stage (a small attention head
// scores every compressed block against the query; the top-k selector keeps the
// best); "Follow the white rabbit: DeepSeek V4's architecture in 3D", indexer
// paragraph (low-precision first pass adapted from V3.2's sparse attention, top
// 1,024 at maximum context); dev.to "How DeepSeek-V4 Achieves Million-Token
// Contexts ...", CSA paragraph (indexer in FP4).
//
// Score of entry j for query n:  d[h] = <q[n,h], k[j]> (MXFP4 x MXFP4, exact in
// fp32), S = fp32 chain acc = fmaf(w[n,h], max(d[h],0), acc) over h = 0..Hi-1.
//
// index_score_kernel -- one CTA per (query, run of entry tiles).  Entries go on the
// MMA M axis (128 per tile), the query's heads on N, the head dim on K:
//   warp 0      TMA producer: 128 FP4 key rows (SWIZZLE_64B) + their scale bytes per stage
//   warp 1      TMEM owner and MMA issuer: rearranges the stage's scale bytes into the
//               tcgen05 scale-factor layout, tcgen05.cp's them to TMEM and issues
//               kind::mxf4.block_scale MMAs into a double-buffered accumulator
//   warps 2..5  epilogue: one thread per entry (TMEM lane), ReLU, head-weighted fp32
//               chain, store of the score row
// topk_kernel -- one CTA per query row: 12/10/10-bit MSB radix select of the k-th
// largest score (order-preserving float->uint key), then an ordered compaction that
// keeps every score above the threshold and the lowest-index ties.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace csa {
namespace {

constexpr int kStages = 8;          // 8 KB key stages
constexpr int kTileE = 128;
constexpr int kMaxTilesPerCta = 31;  // all of a CTA's key scale factors stay in TMEM
constexpr int kIdxThreads = 320;     // producer, MMA, two epilogue groups of four warps
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColSFA = 128;    // 4 columns per tile: [128, 252)
constexpr uint32_t kColSFB = 252;    // 4 columns

struct IndexParams {
  int Nq, Hi, Di, m, B, E_max, E_stride, N;
  int tiles_per_cta, splits;
  const float* w;
  const int32_t* q_pos;
  const int32_t* q_seq;
  const int32_t* n_entries;
  const uint8_t* q_scale;
  float* scores;
  float* score_out;
  int32_t* err;
};

__device__ __forceinline__ int visible_entries(int pos, int m, int n_entries) {
  int v = (pos + 1) / m;
  v = v < 0 ? 0 : v;
  return v < n_entries ? v : n_entries;
}

// kHi: number of indexer heads fixed at compile time (the head chain is straight-line
// code), or 0 to take it from p.Hi at run time.
template <int kHi>
__global__ void __launch_bounds__(kIdxThreads, 2)
    index_score_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ksf,
                       const __grid_constant__ CUtensorMap tm_q, IndexParams p) {
  griddep_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int q = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int seq = p.q_seq[q];
  if (seq < 0 || seq >= p.B) {  // bad sequence id: record it and produce nothing
    if (threadIdx.x == 0 && split == 0) atomicExch(p.err, CSA_DEVERR_INDEX);
    return;
  }
  const int nvis = min(visible_entries(p.q_pos[q], p.m, p.n_entries[seq]), p.E_max);
  const int t_begin = split * p.tiles_per_cta;
  const int t_end = min((nvis + kTileE - 1) / kTileE, t_begin + p.tiles_per_cta);
  const int n_tiles = t_end - t_begin;
  if (n_tiles <= 0) return;  // uniform: nothing allocated yet

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hi = kHi > 0 ? kHi : p.Hi;
  const int row_bytes = p.Di / 2;            // 64 (Di=128) or 32 (Di=64)
  const int a_bytes = kTileE * row_bytes;    // one stage of keys
  const int sf_row = p.Di / 32;              // scale bytes per entry: 4 or 2
  const int sf_bytes = kTileE * sf_row;      // 512 or 256
  const int b_bytes = p.N * row_bytes;
  const uint32_t swz = row_bytes == 64 ? kSwizzle64B : kSwizzle32B;
  const uint32_t sbo = 8 * row_bytes;        // 8-row swizzle atom

  // shared memory carve-up
  uint8_t* sA = smem;                                    // kStages x 8 KB (1024-aligned)
  uint8_t* sB = sA + kStages * 8192;                     // 4 KB
  uint8_t* sSF = sB + 4096;                              // kMaxTilesPerCta x 512: key scales, raw then atom
  uint8_t* sSFB = sSF + kMaxTilesPerCta * 512;           // 512
  float* sW = reinterpret_cast<float*>(sSFB + 512);      // [64] head weights
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + 64);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* b_full = bars + 2 * kStages;
  uint64_t* sf_full = b_full + 1;
  uint64_t* acc_full = sf_full + 1;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(b_full, 1);
    mbar_init(sf_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int tslot = blockIdx.x < 2 ? static_cast<int>(blockIdx.x) : -1;
  if (threadIdx.x == 0) CSA_T(tslot, 0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_ksf);
      prefetch_tmap(&tm_q);
      // every key scale byte of this CTA's tiles, once (they stay in TMEM for the whole run)
      mbar_arrive_expect_tx(sf_full, static_cast<uint32_t>(n_tiles * sf_bytes));
      for (int i = 0; i < n_tiles; ++i)
        tma_load_2d(smem_u32(sSF + i * 512), &tm_ksf, sf_full, 0,
                    (seq * p.E_max + (t_begin + i) * kTileE) * sf_row / 16);
      mbar_arrive_expect_tx(b_full, b_bytes);
      tma_load_2d(smem_u32(sB), &tm_q, b_full, 0, q * Hi);
      for (int it = 0; it < n_tiles; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, p.err, abort_flag)) break;
        const int row = seq * p.E_max + (t_begin + it) * kTileE;
        mbar_arrive_expect_tx(&full[st], a_bytes);
        if (it < 16) CSA_T(tslot, 16 + it);
        tma_load_2d(smem_u32(sA + st * 8192), &tm_k, &full[st], 0, row);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // scale factors of B (the query's heads) into the tcgen05 scale-factor layout:
    // row r -> byte (r % 32) * 16 + (r / 32) * 4 + block; rows >= Hi are zero (2^-127)
    {
      uint32_t words[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        uint32_t v = 0;
        if (r < Hi) {
          const uint8_t* src = p.q_scale + (static_cast<size_t>(q) * Hi + r) * sf_row;
          for (int b = 0; b < sf_row; ++b) v |= static_cast<uint32_t>(src[b]) << (8 * b);
        }
        words[i] = v;
      }
      *reinterpret_cast<uint4*>(sSFB + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc_cp_32x128b_warpx4(tmem + kColSFB, smem_desc(smem_u32(sSFB), 0, 128, kSwizzleNone));
      __syncwarp();
    }
    // key scale factors of all tiles: entry-major bytes -> scale-factor layout (in place per
    // 512-byte slot), then one tcgen05.cp per tile into its own 4 TMEM columns
    bool ok = warp_wait(sf_full, 0, p.err, abort_flag);
    if (ok) {
      for (int i = 0; i < n_tiles; ++i) {
        uint8_t* slot = sSF + i * 512;
        uint32_t words[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j;
          words[j] = sf_row == 4 ? *reinterpret_cast<const uint32_t*>(slot + 4 * r)
                                 : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(slot + 2 * r));
        }
        __syncwarp();
        *reinterpret_cast<uint4*>(slot + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
        __syncwarp();
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        for (int i = 0; i < n_tiles; ++i)
          tc_cp_32x128b_warpx4(tmem + kColSFA + 4 * i, smem_desc(smem_u32(sSF + i * 512), 0, 128, kSwizzleNone));
      __syncwarp();
    }
    ok = ok && warp_wait(b_full, 0, p.err, abort_flag);
    for (int it = 0; ok && it < n_tiles; ++it) {
      const int st = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const int buf = it & 1;
      if (!warp_wait(&full[st], ph, p.err, abort_flag)) break;
      if (lane == 0 && it < 16) CSA_T(tslot, 32 + it);
      if (!warp_wait(&acc_empty[buf], ((it >> 1) & 1) ^ 1, p.err, abort_flag)) break;
      if (lane == 0 && it < 16 && tslot == 0) CSA_T(8, it);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sfa = tmem + kColSFA + 4 * it;
        const uint32_t a0 = smem_u32(sA + st * 8192), b0 = smem_u32(sB);
        for (int kh = 0; kh < p.Di / 64; ++kh) {
          const uint32_t sf_id = 2 * kh;  // byte of the scale column holding blocks 2kh, 2kh+1
          mma_mxf4(tmem + 64 * buf, smem_desc(a0 + 32 * kh, 0, sbo, swz), smem_desc(b0 + 32 * kh, 0, sbo, swz),
                   idesc_mxf4(kTileE, p.N, sf_id, sf_id), kh > 0 ? 1u : 0u, sfa | (sf_id << 30),
                   (tmem + kColSFB) | (sf_id << 30));
        }
        tc_commit(&empty[st]);
        tc_commit(&acc_full[buf]);
        if (it < 16 && tslot == 0) CSA_T(9, it);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    // group 0 (warps 2-5) takes even tiles / accumulator 0, group 1 (warps 6-9) odd tiles
    // / accumulator 1, so two tiles are reduced at once
    const int ew = warp - 2;
    const int grp = ew >> 2;
    const int sub = warp & 3;  // TMEM lane quarter this warp may access
    if (ew * 32 + lane < 64) {
      const int h = ew * 32 + lane;
      sW[h] = h < Hi ? __ldg(p.w + static_cast<size_t>(q) * Hi + h) : 0.f;
    }
    named_bar_sync(1, 256);
    for (int it = grp; it < n_tiles; it += 2) {
      const int buf = grp;
      if (!warp_wait(&acc_full[buf], (it >> 1) & 1, p.err, abort_flag)) break;
      if (sub == 0 && lane == 0 && it < 16 && tslot == 0) CSA_T(6, it);
      tc_fence_after();
      uint32_t acc[64];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + 64 * buf;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (16 * c < Hi) tmem_ld16(taddr + 16 * c, acc + 16 * c);
      tmem_wait_ld();
      if (sub == 0 && lane == 0 && it < 16 && tslot == 0) CSA_T(7, it);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      float s = 0.f;
#pragma unroll
      for (int h = 0; h < 64; h += 4) {
        if (h < Hi) {
          const float4 w4 = *reinterpret_cast<const float4*>(sW + h);
          s = fmaf(w4.x, fmaxf(__uint_as_float(acc[h]), 0.f), s);
          if (h + 1 < Hi) s = fmaf(w4.y, fmaxf(__uint_as_float(acc[h + 1]), 0.f), s);
          if (h + 2 < Hi) s = fmaf(w4.z, fmaxf(__uint_as_float(acc[h + 2]), 0.f), s);
          if (h + 3 < Hi) s = fmaf(w4.w, fmaxf(__uint_as_float(acc[h + 3]), 0.f), s);
        }
      }
      const int e = (t_begin + it) * kTileE + 32 * sub + lane;
      if (sub == 0 && lane == 0 && it < 16) CSA_T(tslot, 48 + it);
      if (e < nvis) {
        p.scores[static_cast<size_t>(q) * p.E_stride + e] = s;
        if (p.score_out) p.score_out[static_cast<size_t>(q) * p.E_max + e] = s;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) CSA_T(tslot, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------- top-k
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
    if (take) out[gt_base + __popc(bgt & lt_mask) + min(eq_before, ties)] = j;
    gt_base += __popc(bgt);
    eq_base += __popc(beq);
  }
  if (threadIdx.x == 0) p.cnt[row] = p.k;
  CSA_T(tslot, 7);
}

int g_index_smem[2][64];
int g_topk_smem[2][64];

}  // namespace

size_t index_workspace_bytes(int Nq, int E_max, int /*k*/) {
  const size_t stride = (static_cast<size_t>(E_max) + 3) & ~size_t(3);
  return static_cast<size_t>(Nq) * stride * sizeof(float) + 256;
}

cudaError_t launch_index_score(const IndexArgs& a, cudaStream_t s) {
  const int row_bytes = a.Di / 2;
  const int N = std::max(16, (a.Hi + 15) / 16 * 16);
  CUtensorMap tm_k, tm_ksf, tm_q;
  const CUtensorMapSwizzle swz = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!encode_2d_u8(&tm_k, a.k_fp4, row_bytes, static_cast<uint64_t>(a.B) * a.E_max, row_bytes, kTileE, swz))
    return cudaErrorInvalidValue;
  const uint64_t sf_total = static_cast<uint64_t>(a.B) * a.E_max * (a.Di / 32);
  if (!encode_2d_u8(&tm_ksf, a.k_scale, 16, sf_total / 16, 16, kTileE * (a.Di / 32) / 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tm_q, a.q_fp4, row_bytes, static_cast<uint64_t>(a.Nq) * a.Hi, row_bytes, N, swz))
    return cudaErrorInvalidValue;

  IndexParams p{};
  p.Nq = a.Nq;
  p.Hi = a.Hi;
  p.Di = a.Di;
  p.m = a.m;
  p.B = a.B;
  p.E_max = a.E_max;
  p.E_stride = a.E_stride;
  p.N = N;
  const int tiles_max = (a.E_max + kTileE - 1) / kTileE;
  int splits = std::max(1, std::min(tiles_max, 2 * num_sms() / std::max(1, a.Nq)));
  splits = std::max(splits, (tiles_max + kMaxTilesPerCta - 1) / kMaxTilesPerCta);
  p.tiles_per_cta = (tiles_max + splits - 1) / splits;
  p.splits = (tiles_max + p.tiles_per_cta - 1) / p.tiles_per_cta;
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.q_seq = a.q_seq;
  p.n_entries = a.n_entries;
  p.q_scale = a.q_scale;
  p.scores = a.scores_ws;
  p.score_out = a.score_out;
  p.err = device_error_word();

  const size_t smem = 1024 + kStages * 8192 + 4096 + kMaxTilesPerCta * 512 + 512 + 256 + 512;
  if (a.Hi == 64) {
    cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(index_score_kernel<64>), smem, g_index_smem[0]);
    if (e != cudaSuccess) return e;
    return launch_pdl(index_score_kernel<64>, dim3(a.Nq * p.splits), dim3(kIdxThreads), smem, s, tm_k, tm_ksf, tm_q, p);
  }
  cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(index_score_kernel<0>), smem, g_index_smem[1]);
  if (e != cudaSuccess) return e;
  return launch_pdl(index_score_kernel<0>, dim3(a.Nq * p.splits), dim3(kIdxThreads), smem, s, tm_k, tm_ksf, tm_q, p);
}

cudaError_t launch_topk_select(const IndexArgs& a, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
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
  const bool big = a.E_max > 4096;
  // dynamic limit leaves room for the kernel's static shared memory
  const int max_dyn = 227 * 1024 - 1024;
  const int cache_cap = std::min(a.E_max, (max_dyn - (4096 + 8192) * 4) / 4);
  t.cache_cap = cache_cap;
  const size_t tsmem = (4096 + 8192 + static_cast<size_t>(cache_cap)) * 4;
  if (big) {
    e = set_dyn_smem(reinterpret_cast<const void*>(topk_kernel<1024>), tsmem, g_topk_smem[1]);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_kernel<1024>, dim3(a.Nq), dim3(1024), tsmem, s, t);
  } else {
    e = set_dyn_smem(reinterpret_cast<const void*>(topk_kernel<256>), tsmem, g_topk_smem[0]);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_kernel<256>, dim3(a.Nq), dim3(256), tsmem, s, t);
  }
  return cudaGetLastError();
}

}  // namespace csa
