// topk.cu -- exact top-k selection of indexer scores, ties to the lowest index, output
// in ascending index order (padded with -1 when fewer than k entries are visible).
//
// Sources: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
// §2.3 (the selector keeps the k best-scoring compressed entries) and §4 (k = 512 /
// 1024); "Follow the white rabbit: DeepSeek V4's architecture in 3D", indexer paragraph
// (top 1,024 entries at maximum context).
//
// Two kernels compute the same result:
//   topk_reg_kernel<C, ...>  the row held in registers by a thread-block cluster of C
//                            CTAs (few rows: decode; each CTA owns a contiguous slice and
//                            the CTAs exchange ranges, histograms, member keys and counts
//                            through distributed shared memory), or by one CTA (C = 1:
//                            many rows, up to 32768 entries)
//   topk_kernel              one CTA per row staged in shared memory (longer rows)
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
#include "topk_regs.cuh"

namespace csa {
namespace {

__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t peers = __match_any_sync(0xffffffffu, active ? bin : 0xFFFFFFFFu);
  if (active && (threadIdx.x & 31) == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
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


// The row from global memory into registers, then topk_regs_row (a cluster of C CTAs per
// row when C > 1).
template <int C, int THREADS, int EPT>
__global__ void __launch_bounds__(THREADS) topk_reg_kernel(TopkParams p) {
  using Mask = TopkMask<EPT>;
  constexpr Mask kOne = 1;
  constexpr int kSlice = THREADS * EPT;  // entries per CTA
  griddep_enter();
  const int rank = static_cast<int>(blockIdx.x % C);  // == %cluster_ctarank for 1-D clusters
  const int row = static_cast<int>(blockIdx.x / C);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seq = p.q_seq[row];
  const int nv = (seq < 0 || seq >= p.B) ? 0 : min(visible_entries(p.q_pos[row], p.m, p.n_entries[seq]), p.E_max);
  if (nv <= p.k) {  // the same for every CTA of the cluster: none reaches a cluster barrier
    int32_t* out = p.idx + static_cast<size_t>(row) * p.k;
    if (rank == 0) {
      for (int j = threadIdx.x; j < p.k; j += THREADS) out[j] = j < nv ? j : -1;
      if (threadIdx.x == 0) p.cnt[row] = nv;
    }
    return;
  }
  const int tslot = (row < 2 && rank == 0 && threadIdx.x == 0) ? 2 + row : -1;
  (void)tslot;  // phase stamps only in timing builds
  CSA_T(tslot, 0);

  // ---- this CTA's slice into registers
  const int wbase = rank * kSlice + 32 * EPT * warp;
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
  topk_regs_row<C, THREADS, EPT>(p, row, rank, v, valid);
}

int g_topk_smem[2][64];

// Whether Nq clusters of 16 CTAs of 1024 threads can be resident at once (a cluster of 16
// needs 16 free SMs in one GPC); the answer per device is cached.
bool topk_cluster16_fits(int Nq) {
  static int max_clusters[64];  // 0: not asked yet, -1: none
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (max_clusters[dev] == 0) {
    int n = 0;
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(topk_reg_kernel<16, 1024, 16>),
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(1024);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(topk_reg_kernel<16, 1024, 16>), &cfg) !=
          cudaSuccess)
        n = 0;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    max_clusters[dev] = n > 0 ? n : -1;
  }
  return max_clusters[dev] >= Nq;
}

// one cluster of C CTAs (1024 threads each) per row, the fewest entries per thread that hold the row
template <int C>
cudaError_t launch_topk_cluster(const TopkParams& t, int Nq, int E_max, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(Nq * C)), block(1024);
  if constexpr (C == 16) {  // a non-portable cluster size: rows of up to 16 x 1024 x 16 entries
    static int allowed[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !allowed[dev]) {
      const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(topk_reg_kernel<16, 1024, 16>),
                                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      allowed[dev] = 1;
    }
    return launch_pdl_cluster(topk_reg_kernel<16, 1024, 16>, grid, block, 0, C, s, t);
  } else {
  if (E_max <= C * 1024 * 8) return launch_pdl_cluster(topk_reg_kernel<C, 1024, 8>, grid, block, 0, C, s, t);
  if (E_max <= C * 1024 * 16) return launch_pdl_cluster(topk_reg_kernel<C, 1024, 16>, grid, block, 0, C, s, t);
  return launch_pdl_cluster(topk_reg_kernel<C, 1024, 32>, grid, block, 0, C, s, t);
  }
}

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
  // Few rows longer than 2048 entries: a cluster of C CTAs per row, C as large as one wave
  // of CTAs (one per SM) allows and the cluster's registers hold the row.
  int C = 0;
  if (a.E_max > 2048) {
    // 16 CTAs (a non-portable cluster) only for rows beyond 8 x 1024 x 16 entries (the
    // 1M-context decode), and only where 16-CTA clusters can be resident at once
    if (a.E_max > 8 * 1024 * 16 && a.E_max <= 16 * 1024 * 16 && static_cast<int64_t>(a.Nq) * 16 <= num_sms() &&
        topk_cluster16_fits(a.Nq))
      C = 16;
    for (int c = 8; c >= 2 && C == 0; c >>= 1)
      if (static_cast<int64_t>(a.Nq) * c <= num_sms() && static_cast<int64_t>(c) * 1024 * 32 >= a.E_max) C = c;
  }
  if (C == 16) {
    e = launch_topk_cluster<16>(t, a.Nq, a.E_max, s);
  } else if (C == 8) {
    e = launch_topk_cluster<8>(t, a.Nq, a.E_max, s);
  } else if (C == 4) {
    e = launch_topk_cluster<4>(t, a.Nq, a.E_max, s);
  } else if (C == 2) {
    e = launch_topk_cluster<2>(t, a.Nq, a.E_max, s);
  } else if (a.E_max <= 2048) {  // one CTA per row, the row in registers
    e = launch_pdl(topk_reg_kernel<1, 128, 16>, dim3(a.Nq), dim3(128), 0, s, t);
  } else if (a.E_max <= 8192) {
    e = launch_pdl(topk_reg_kernel<1, 256, 32>, dim3(a.Nq), dim3(256), 0, s, t);
  } else if (a.E_max <= 32768) {
    e = launch_pdl(topk_reg_kernel<1, 1024, 32>, dim3(a.Nq), dim3(1024), 0, s, t);
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
