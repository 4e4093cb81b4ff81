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
//   O^T[512 d, 64 heads]    += V^T[512 x 128] . P^T         (V^T read MN-major, P^T MN-major)
// with K = V (shared KV).
//
// A tile's 128 rows arrive slab by slab (a slab = 64 of the 512 dims x 128 rows = 16 KB,
// SWIZZLE_128B), gathered with cp.async or, for a contiguous run of rows, as a TMA box.
// Two pipelines:
//   * attend (shares longer than three tiles: prefill) keeps a tile resident: its eight
//     slabs fill eight slots (the ring and the first two P buffers), QK reads them, the
//     softmax writes P into the third P buffer, and PV reads the same slots as V, each
//     128-dim chunk then releasing its two slots to the next tile -- every key row is
//     loaded once.  The softmax keeps a running max that only moves when a tile raises it
//     by more than 2^8 (then O^T is rescaled in TMEM).
//   * attend_2pass (at most three tiles: decode splits) streams every tile's K slabs from
//     HBM through a 9-slot ring with S^T of each tile kept in TMEM, runs one exact
//     softmax, then re-gathers the rows (now in L2) for PV.
// S^T takes 64 TMEM columns per tile buffer, O^T 4 x 64.  (At M = 128, N = 64 heads a QK
// MMA of K = 16 costs ~75 cycles and a PV MMA ~64: about half the bf16 rate, whatever the
// pipeline; loading each row once measured 7 % faster than re-reading it for PV.)
//
// Roles (416 threads): warps 0-7 softmax + epilogue, warps 8-11 producers (cp.async
// gathers of 16-byte chunks, TMA boxes; Q arrives by TMA), warp 12 TMEM owner and MMA
// issuer.  Sums over keys stay per thread and are reduced once at the end.
// With one CTA per query the window starts on a tile boundary (when that adds no tile),
// so a full tile of HCA entries or of window rows is one contiguous run of 128 rows: its
// slabs arrive as 2-D TMA boxes instead of row gathers.
// When a query's keys are split over several CTAs (few queries), the splits of a
// query form a thread-block cluster: each CTA writes an
// unnormalised fp32 partial and its (max, sum) to the workspace, the cluster
// synchronises, and CTA r combines heads [r H/S, (r+1) H/S) of the query.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>

#include "internal.h"
#include "ptx.cuh"
#include "rowprep.cuh"
#include "tmap.h"

namespace csa {
namespace {

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kBN = 128;            // keys per tile
constexpr int kSlabs = 8;           // 64-dim slabs per tile
constexpr int kSlabBytes = 16384;
constexpr int kRing = 6;            // even: the two slabs of a 128-dim PV chunk sit in adjacent slots
constexpr int kProdWarps = 4;                          // gather producers
static_assert(kBN == 32 * kProdWarps, "one row of a tile per producer lane");
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kMmaWarp = 8 + kProdWarps;               // TMEM owner and MMA issuer
constexpr int kAttnThreads = 32 * (kMmaWarp + 1);      // 8 softmax warps first
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;       // 2 x 64 columns
constexpr uint32_t kColO = 128;     // 4 x 64 columns
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kSplitSMs = 148;             // B200 SM count used to size decode splits
constexpr int kMaxSplits = 8;              // portable cluster size

constexpr int kPBufs = 3;           // P buffers: the two-pass pipeline uses 3; attend holds slabs in 2 and P in the third
constexpr int kMaxTiles2 = kPBufs;  // tiles a CTA's share may have on the two-pass pipeline
constexpr uint32_t kColO2 = 256;    // two-pass: S^T of up to 3 tiles in [0, 192), O^T in [256, 512)
// Two-pass slab slots: the K pass cycles through the ring and the P buffers (the softmax
// writes P only after the last QK), the V pass through the ring and Q's four 16 KB slabs
// (free once the last QK has completed).  Barrier pairs: K slot s and V slot s < kRing
// share pair s; V slot kRing + i uses pair kRing + kPBufs + i.
constexpr int kSlotsK2 = kRing + kPBufs;
constexpr int kSlotBars = kRing + kPBufs + 4;
constexpr size_t kOffQ = 0;                                       // 64 KB: [8 d-atoms][64 heads][128 B]
constexpr size_t kOffRing = 64 * 1024;                            // kRing x 16 KB
constexpr size_t kOffP = kOffRing + kRing * kSlabBytes;           // kPBufs x 16 KB: [128 keys][128 B]
constexpr size_t kOffSmall = kOffP + kPBufs * 16384;              // reductions, stats, barriers
// reductions and stats (832 floats), rope table (32 float2), row flags, 40 barriers, TMEM
// slot and abort flag, laid out by AttnSmem below
constexpr size_t kSmallUsed = 832 * 4 + 32 * 8 + 128 * kPBufs + (1 + 2 * kSlotBars + kPBufs + 2 + 2 + 1 + kPBufs + 4) * 8 + 8;
constexpr size_t kOffIdx = kOffSmall + 5120;                      // this CTA's slice of the index list
static_assert(kSmallUsed <= 5120, "small shared-memory region");
constexpr int kIdxCap = 2048;
constexpr size_t kAttnSmem = kOffIdx + 4 * kIdxCap + 1024;        // + alignment slack
static_assert(kAttnSmem <= 227 * 1024, "shared memory budget");
static_assert(kRing % 2 == 0, "ring shape");

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
  int two_pass;    // every CTA's share is at most kMaxTiles2 tiles: attend_2pass
  int persist;     // splits == 1 and attend: persistent CTAs take queries blockIdx.x, + gridDim.x, ...
  int align;       // tile-aligned key list: the window starts on a tile boundary
  int tma_e;       // dense mode, entries tensor map valid: full entry tiles load by TMA
  int tma_w;       // window tensor map valid: full window tiles load by TMA
  int q_prep;      // q is raw: RMSNorm (q_norm) and partial RoPE are applied as it is loaded
  int q_norm, rope_dims;
  float q_eps, rope_theta;
  int32_t* err;
};

// A query's key list: n_sel entries (rows [0, n_sel)), then n_win window rows (rows
// [win0, win0 + n_win)).  On the tile-aligned layout win0 is n_sel rounded up to a whole
// tile when that costs no extra tile, so that every tile holds rows of one contiguous run;
// rows [n_sel, win0) have no source.
struct KeyList {
  int b, n_sel, n_win, win0;
  int64_t u_lo, wbase;
};

// The query's step metadata: its sequence (in range or not), position, window base and
// (dense mode) entry count.  No kernel of this library writes these arrays, and a kernel
// of the caller's that does never lets this one start before it completes (it does not
// release its dependents early), so they are read before the wait on the previous grid.
struct KeyMeta {
  bool ok;
  int b;
  int64_t t, wbase, ne;
};

__device__ __forceinline__ KeyMeta key_meta(const AttnParams& p, int n) {
  KeyMeta m{};
  m.b = p.q_seq[n];
  m.ok = m.b >= 0 && m.b < p.B;
  if (m.ok) {
    m.t = p.q_pos[n];
    m.wbase = p.window_base[m.b];
    m.ne = p.dense ? p.n_entries[m.b] : 0;
  }
  return m;
}

// The key list; in sparse mode the selection count comes from the previous grid (top-k),
// so this runs after the wait.
__device__ __forceinline__ KeyList key_list(const AttnParams& p, int n, const KeyMeta& m) {
  KeyList kl;
  kl.b = m.b;
  const int64_t t = m.t;
  if (p.dense) {
    int64_t v = (t + 1) / p.mprime;
    v = v < 0 ? 0 : v;
    const int64_t ne = min(m.ne, static_cast<int64_t>(p.E_max));
    kl.n_sel = static_cast<int>(v < ne ? v : ne);
  } else {
    const int c = p.cnt ? p.cnt[n] : 0;
    kl.n_sel = c < 0 ? 0 : (c > p.k ? p.k : c);
  }
  kl.wbase = m.wbase;
  int64_t lo = t - p.W + 1;
  if (lo < 0) lo = 0;
  if (lo < kl.wbase) lo = kl.wbase;
  int64_t hi = t;
  if (hi > kl.wbase + p.Tw - 1) hi = kl.wbase + p.Tw - 1;
  kl.u_lo = lo;
  kl.n_win = (p.W > 0 && hi >= lo) ? static_cast<int>(hi - lo + 1) : 0;
  kl.win0 = kl.n_sel;
  if (p.align) {
    const int padded = (kl.n_sel + kBN - 1) / kBN * kBN;
    const int tiles_a = padded / kBN + (kl.n_win + kBN - 1) / kBN;
    const int tiles_u = (kl.n_sel + kl.n_win + kBN - 1) / kBN;
    if (tiles_a <= tiles_u) kl.win0 = padded;
  }
  return kl;
}

// A tile (rows [ts, ts + kBN) of the key list) whose rows are all present and form one
// contiguous run of a tensor -- every row a dense-mode entry, or every row a window row --
// loads slab by slab as 2-D TMA boxes of 128 rows x 128 bytes.  Returns the tensor map
// and the first row's coordinate in it, or no map (the rows are gathered).  Ragged tiles
// are always gathered: their missing rows must read as zeros, which a box cannot promise.
struct TileBox {
  const CUtensorMap* map;
  int row;
};

__device__ __forceinline__ TileBox tile_box(const AttnParams& p, const KeyList& kl, const CUtensorMap& tm_e,
                                            const CUtensorMap& tm_w, int ts, int row_end) {
  TileBox tb{nullptr, 0};
  if (!p.align || ts + kBN > row_end) return tb;
  if (ts + kBN <= kl.n_sel) {
    if (p.tma_e) tb = TileBox{&tm_e, kl.b * p.E_max + ts};
  } else if (ts >= kl.win0) {
    if (p.tma_w) tb = TileBox{&tm_w, kl.b * p.Tw + static_cast<int>(kl.u_lo + (ts - kl.win0) - kl.wbase)};
  }
  return tb;
}

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {  // byte offset inside an 8-row x 128 B atom column
  return static_cast<uint32_t>(row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// Row of a tile that lane `l` of gather warp `w` (0-3) owns: a warp takes 32 consecutive
// rows of the key list (sorted selections put neighbouring entries in one warp's copies),
// and gather_warp is the owner of a row.
__device__ __forceinline__ int gather_row(int w, int l) { return 32 * w + l; }
__device__ __forceinline__ int gather_warp(int row) { return row / 32; }

// Source of row g of query n's key list: a selected entry (g < n_sel), a window row
// (g >= win0), or nothing (past row_end, the alignment gap, or an index outside the
// cache, which sets the device error word when `flag`).  `sidx` (nullable) is the CTA's
// staged slice of the index list, starting at row_begin.
__device__ __forceinline__ const uint16_t* key_row_src(const AttnParams& p, const KeyList& kl, int n, int g,
                                                       int row_begin, int row_end, const int32_t* sidx,
                                                       bool flag) {
  if (g >= row_end) return nullptr;
  if (g < kl.n_sel) {
    const int e = p.dense ? g : (sidx != nullptr ? sidx[g - row_begin] : p.idx[static_cast<size_t>(n) * p.k + g]);
    if (e >= 0 && e < p.E_max) return p.entries + (static_cast<size_t>(kl.b) * p.E_max + e) * kD;
    if (flag) atomicExch(p.err, CSA_DEVERR_INDEX);
    return nullptr;
  }
  if (g < kl.win0) return nullptr;
  const int64_t u = kl.u_lo + (g - kl.win0);
  return p.window + (static_cast<size_t>(kl.b) * p.Tw + static_cast<size_t>(u - kl.wbase)) * kD;
}

// Slab ka of a tile (64 dims of its 128 rows) into `dst`, by a group of four warps whose
// lane l of warp w holds the source of row gather_row(w, l) (src_ll; valid = false: no
// row, zero-filled): one TMA box when the tile is a contiguous block, else 16-byte
// cp.async chunks.  `bar` takes 128 arrivals per slab: with a box, lane 0 of each warp
// makes its warp's 32 at once (the first with the byte count); with cp.async, every
// thread arrives once its own copies have landed.
__device__ __forceinline__ void gather_slab(uint32_t dst, const TileBox& box, int ka, unsigned long long src_ll,
                                            bool valid, int w, int lane, uint64_t* bar) {
  if (box.map != nullptr) {
    if (lane == 0) {
      if (w == 0) {
        mbar_arrive_expect_tx(bar, kSlabBytes);
        tma_load_2d(dst, box.map, bar, ka * 128, box.row);
        mbar_arrive_cnt(bar, 31);
      } else {
        mbar_arrive_cnt(bar, 32);
      }
    }
    return;
  }
#pragma unroll
  for (int qb = 0; qb < 256; qb += 32) {  // chunk q: 16 bytes q % 8 of the row of lane q / 8
    const int q = qb + lane;
    const int rl = q >> 3, c = q & 7;
    const uint16_t* rs = reinterpret_cast<const uint16_t*>(__shfl_sync(0xffffffffu, src_ll, rl));
    const bool rv = __shfl_sync(0xffffffffu, valid, rl);
    cp_async_16(dst + sw128(gather_row(w, rl), c), rs + (ka * 8 + c) * 8, rv);
  }
  cp_async_mbar_arrive_noinc(bar);
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

// 2^x by the hardware approximation (relative error ~2^-22; probabilities are rounded to
// bf16 right after)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory layout of a CTA (one definition for the set-up and the pipeline).
struct AttnSmem {
  uint8_t* sQ;
  uint8_t* sRing;
  uint8_t* sP;
  float* red_max;    // [4][64]
  float* red_sum;    // [4][64]
  float* m_run;      // [64]
  float* l_run;      // [64]
  float* alpha;      // [64]
  float* inv_l;      // [64]
  float* hscale;     // [64]: logit scale per head (log2 units; with the query's norm folded in)
  float2* cs_tab;    // [32]: (cos, sin) of the query's rope pairs (query preparation)
  uint8_t* row_ok;   // [kPBufs][128]: key row has a valid source
  uint64_t* q_full;     // TMA: Q landed
  uint64_t* full;       // [kSlotBars] producers: slab landed
  uint64_t* slot_free;  // [kSlotBars] MMA commit: slab consumed
  uint64_t* s_full;     // [kPBufs] MMA commit: S^T of a tile in TMEM
  uint64_t* s_free;     // [2] softmax warps: S^T read
  uint64_t* p_full;     // [2] softmax warps: P written (and O^T rescaled)
  uint64_t* o_done;     // MMA commit: PV of a tile complete
  uint64_t* row_ready;  // [kPBufs] producers: row_ok of a tile written
  uint64_t* fin;        // MMA commit: every MMA of the CTA complete
  uint64_t* q_ready;    // softmax warps: the query prepared in place (query preparation only)
  uint64_t* q_free;     // Q's slabs may be reloaded: the query's last QK completed (MMA commit) and
                        // the softmax threads read Q for the last time (query preparation)
  uint64_t* o_free;     // softmax warps: O^T of a query read from TMEM (the next query may overwrite it)
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  int32_t* sidx;        // this CTA's slice of the index list
  __device__ explicit AttnSmem(uint8_t* smem) {
    sQ = smem + kOffQ;
    sRing = smem + kOffRing;
    sP = smem + kOffP;
    red_max = reinterpret_cast<float*>(smem + kOffSmall);
    red_sum = red_max + 256;
    m_run = red_sum + 256;
    l_run = m_run + 64;
    alpha = l_run + 64;
    inv_l = alpha + 64;
    hscale = inv_l + 64;
    cs_tab = reinterpret_cast<float2*>(hscale + 64);
    row_ok = reinterpret_cast<uint8_t*>(cs_tab + 32);
    uint64_t* bars = reinterpret_cast<uint64_t*>(row_ok + 128 * kPBufs);
    q_full = bars;
    full = q_full + 1;
    slot_free = full + kSlotBars;
    s_full = slot_free + kSlotBars;
    s_free = s_full + kPBufs;
    p_full = s_free + 2;
    o_done = p_full + 2;
    row_ready = o_done + 1;
    fin = row_ready + kPBufs;
    q_ready = fin + 1;
    q_free = q_ready + 1;
    o_free = q_free + 1;
    tmem_slot = reinterpret_cast<uint32_t*>(o_free + 1);
    abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    sidx = reinterpret_cast<int32_t*>(smem + kOffIdx);
  }
};

// The query prepared in the kernel, off the MMA's critical path.  The raw query lands in
// sQ by TMA as usual and QK starts on it at once; the preparation only has to finish the
// part that differs:
//   * RoPE rotates the last rope_dims channels (all in Q's last 64-dim atom, rope_dims <=
//     64) in place; the MMA waits for them (q_ready) only before the first QK of that atom;
//   * RMSNorm scales head row h by inv_h, which scales S^T's column h by inv_h: the softmax
//     folds it into the logit scale (hscale[h] = scale log2(e) inv_h), computed while QK
//     runs, instead of Q being rescaled.
// Mathematically the query csa_norm_rope would write (a rotation commutes with a scale);
// the rounding differs: the rotated channels are rounded to bf16 unscaled and the scale
// is applied in float32.  The 256 softmax threads split the work as (head h = t / 4,
// quarter c = t % 4): in the last atom, chunks 2c and 2c + 1 of row h (16 channels); for
// the norm, 112 channels of atoms 0..6 plus those 16.  cs_tab holds the (cos, sin) of the
// query's rope pairs; ssq the per-thread sums of squares of the raw last-atom channels.
__device__ __forceinline__ void prep_query(const AttnParams& p, int n, uint8_t* sQ, uint64_t* q_full, uint32_t q_ph,
                                           uint64_t* q_ready, float* hscale, float2* cs_tab,
                                           volatile int* abort_flag, int warp, int lane) {
  const int t = static_cast<int>(threadIdx.x);  // 0..255 (softmax warps)
  const int h = t >> 2, c = t & 3;
  const int npairs = p.rope_dims >> 1;
  const int rope_base = kD - p.rope_dims;  // >= 448: inside the last atom
  if (warp == 0 && lane < npairs)  // overlaps the query's load
    cs_tab[lane] = rowprep::rope_cs(static_cast<double>(p.q_pos[n]), rowprep::inv_freq(p.rope_theta, lane, p.rope_dims));
  const bool got = warp_wait(q_full, q_ph, p.err, abort_flag);
  named_bar_sync(1, 256);  // cs_tab written
  float ss = 0.f;
  if (got) {
    // last atom: 16 raw channels [448 + 16 c, 448 + 16 c + 16) of row h, rotated in place
    uint8_t* a7 = sQ + 7 * 8192;
    uint4* p0 = reinterpret_cast<uint4*>(a7 + sw128(h, 2 * c));
    uint4* p1 = reinterpret_cast<uint4*>(a7 + sw128(h, 2 * c + 1));
    const uint4 r0 = *p0, r1 = *p1;
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) ss = fmaf(v[e], v[e], ss);
    if (npairs > 0 && 448 + 16 * c + 16 > rope_base) {
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const int d = 448 + 16 * c + e;
        if (d >= rope_base) {
          const float2 cs = cs_tab[(d - rope_base) >> 1];
          const float x0 = v[e], x1 = v[e + 1];
          v[e] = fmaf(x0, cs.x, -(x1 * cs.y));
          v[e + 1] = fmaf(x0, cs.y, x1 * cs.x);
        }
      }
      *p0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
      *p1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                       pack_bf16x2(v[14], v[15]));
      fence_proxy_async_smem();
    }
  }
  mbar_arrive(q_ready);
  if (got) {
    // the norm: 112 raw channels of atoms 0..6 (chunks 14 c .. 14 c + 13 of row h) while QK runs
#pragma unroll 7
    for (int k = 0; k < 14; ++k) {
      const int ch = 14 * c + k;  // chunk index over atoms 0..6: atom ch / 8, chunk ch % 8
      const uint4 r = *reinterpret_cast<const uint4*>(sQ + (ch >> 3) * 8192 + sw128(h, ch & 7));
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
        ss = fmaf(lo, lo, ss);
        ss = fmaf(hi, hi, ss);
      }
    }
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);  // the four threads of row h are lanes 4k .. 4k + 3
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  if (c == 0) hscale[h] = p.scale_log2 * (p.q_norm ? 1.0f / sqrtf(ss / static_cast<float>(kD) + p.q_eps) : 1.f);
}

// One CTA's share of a query: rows [row_begin, row_end) of its key list, n_tiles > 0.
// Writes the normalised output (splits == 1) or the unnormalised partial + (max, sum).
// A CTA may take several queries in turn (persistent CTAs): qi counts the queries this CTA
// took before this one, T0 their tiles, so that every barrier's phase continues; the
// roles do not wait for one another between queries (the next query's loads and QK run
// while the softmax warps write this one's output).
__device__ __forceinline__ void attend(const AttnParams& p, const CUtensorMap& tm_q, const CUtensorMap& tm_e,
                                       const CUtensorMap& tm_w, uint8_t* smem, uint32_t tmem, int n, int split,
                                       const KeyList& kl, int row_begin, int row_end, int n_tiles, int qi,
                                       int T0) {
  const AttnSmem L(smem);
  uint8_t* sQ = L.sQ;
  uint8_t* sRing = L.sRing;
  uint8_t* sP = L.sP;
  float* red_max = L.red_max;
  float* red_sum = L.red_sum;
  float* m_run = L.m_run;
  float* l_run = L.l_run;
  float* alpha = L.alpha;
  float* inv_l = L.inv_l;
  uint8_t* row_ok = L.row_ok;
  uint64_t* q_full = L.q_full;
  uint64_t* full = L.full;
  uint64_t* slot_free = L.slot_free;
  uint64_t* s_full = L.s_full;
  uint64_t* s_free = L.s_free;
  uint64_t* p_full = L.p_full;
  uint64_t* o_done = L.o_done;
  uint64_t* row_ready = L.row_ready;
  uint64_t* fin = L.fin;
  volatile int* abort_flag = L.abort_flag;
  int32_t* sidx = L.sidx;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int tslot = blockIdx.x < 2 ? 4 + static_cast<int>(blockIdx.x) : -1;
  if (threadIdx.x == 0) CSA_T(tslot, 0);
  CSA_TB(2);

  if (warp >= 8 && warp < 8 + kProdWarps) {
    // ------------------------------------------------------------ gather producers
    // Lane l of producer warp pw owns row gather_row(pw, l) of every tile and resolves its
    // source; the warp issues the 8 x 16-byte chunks per slab of its 32 rows.  The warps
    // never wait on one another, so one that gives up cannot stall the others.
    const int pw = warp - 8;
    const int ptid = threadIdx.x - 256;
    const int my_row = gather_row(pw, lane);
    // query: 64 head rows x 1 KB as 8 boxes of 64 rows x 128 B (one per 64-dim atom), once
    // the previous query's last QK has released Q's slabs
    if (ptid == 0 && (qi == 0 || mbar_wait(L.q_free, (qi - 1) & 1, p.err, abort_flag))) {
      mbar_arrive_expect_tx(q_full, kH * kD * 2);
      for (int a = 0; a < 8; ++a) tma_load_2d(smem_u32(sQ + a * 8192), &tm_q, q_full, 128 * a, n * kH);
    }
    // this CTA's slice of the index list, staged once per warp (no dependent global load
    // per row); each warp copies the part its own lanes will read (they finished reading
    // the previous query's slice: their last gathers were issued)
    const int sel_here = max(0, min(row_end, kl.n_sel) - row_begin);
    const bool staged = !p.dense && sel_here <= kIdxCap;
    if (staged)
      for (int i = lane; i < sel_here; i += 32)
        if (gather_warp(i % kBN) == pw) sidx[i] = p.idx[static_cast<size_t>(n) * p.k + row_begin + i];
    __syncwarp();
    bool ok = true;
    int j = 0;  // slab sequence number
    // tile t's slab ka goes into slot ka (the ring and the first two P buffers: eight
    // contiguous 16 KB slots), phase t & 1
    for (int tile = 0; ok && tile < n_tiles; ++tile) {
      // source of this lane's row (invalid indices are flagged once)
      const int ts = row_begin + tile * kBN;
      const uint16_t* src_row = key_row_src(p, kl, n, ts + my_row, row_begin, row_end, staged ? sidx : nullptr, true);
      const bool valid = src_row != nullptr;
      const unsigned long long src_ll = reinterpret_cast<unsigned long long>(valid ? src_row : p.entries);
      const TileBox box = tile_box(p, kl, tm_e, tm_w, ts, row_end);
      const int T = T0 + tile;  // the CTA's tile count: phases continue across its queries
      for (int ka = 0; ka < kSlabs; ++ka, ++j) {
        const int slot = ka;
        if (!warp_wait(&slot_free[slot], (T & 1) ^ 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        if (ptid == 0 && tslot == 4 && j < 64) CSA_T(10, j);
        if (ka == 0) {
          // the softmax of the tile two back (same buffer) finished before this slot freed
          row_ok[(T & 1) * 128 + my_row] = valid ? 1 : 0;
          mbar_arrive(&row_ready[T & 1]);
          if (ptid == 0 && tile < 8) CSA_T(tslot, 8 + tile);
        }
        // the slab's barrier completes when every producer thread's copies have landed;
        // the consumer fences the async proxy after its wait
        gather_slab(smem_u32(sRing + slot * kSlabBytes), box, ka, src_ll, valid, pw, lane, &full[slot]);
      }
    }
    cp_async_wait_all();  // nothing in flight when the CTA exits
    {  // Q must have landed before the CTA may exit (already true on the normal path)
      volatile int never = 0;
      if (ptid == 0) mbar_wait(q_full, qi & 1, p.err, &never);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, kH, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, kH, true, true);
    const uint32_t q0 = smem_u32(sQ), ring0 = smem_u32(sRing), p0 = smem_u32(sP);
    bool ok = warp_wait(q_full, qi & 1, p.err, abort_flag);
    // query preparation: the rotated atoms are ready for the MMA once q_ready completes
    const int rope_atom = p.q_prep && p.rope_dims > 0 ? (kD - p.rope_dims) / 64 : kSlabs;
    bool q_ready_seen = rope_atom >= kSlabs;
    int j = 0;
    // QK(t) from slots 0..7, then (once P(t) is written) PV(t) from the same slots, each
    // 128-dim chunk releasing its two slots to tile t + 1; P in the third P buffer
    for (int tile = 0; ok && tile < n_tiles; ++tile) {
      const int T = T0 + tile;
      const int b = T & 1;
      if (T >= 2 && !warp_wait(&s_free[b], ((T - 2) >> 1) & 1, p.err, abort_flag)) break;
      for (int ka = 0; ka < kSlabs; ++ka, ++j) {
        if (!warp_wait(&full[ka], T & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        if (!q_ready_seen && ka >= rope_atom) {  // the query's rotated channels are written
          q_ready_seen = true;
          if (!warp_wait(L.q_ready, qi & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
        }
        if (lane == 0 && tslot == 4 && j < 64) CSA_T(12, j);
        fence_proxy_async_smem();  // the producers' cp.async writes, seen through the barrier
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColS + 64 * b, smem_desc(ring0 + ka * kSlabBytes + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(q0 + ka * 8192 + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, (ka | kk) ? 1u : 0u);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(&s_full[b]);
        if (tile == n_tiles - 1) tc_commit(L.q_free);  // Q's slabs are read by no later MMA
        if (tile < 8) CSA_T(tslot, 24 + tile);
      }
      __syncwarp();
      if (!warp_wait(&p_full[b], (T >> 1) & 1, p.err, abort_flag)) break;
      // the first PV of a query overwrites O^T: the previous query's epilogue must have read it
      if (tile == 0 && qi > 0 && !warp_wait(L.o_free, (qi - 1) & 1, p.err, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + kColO + 64 * dc,
                     smem_desc(ring0 + 2 * dc * kSlabBytes + ks * 2048, kSlabBytes, 1024, kSwizzle128B),
                     smem_desc(p0 + 2 * 16384 + ks * 2048, 16384, 1024, kSwizzle128B), idesc_pv,
                     (tile > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&slot_free[2 * dc]);
          tc_commit(&slot_free[2 * dc + 1]);
        }
        tc_commit(o_done);
        if (tile < 8) CSA_T(tslot, 32 + tile);
      }
      __syncwarp();
    }
    // o_done may have two phases outstanding when the softmax finishes its last tile, so
    // the epilogue waits on a barrier of its own
    if (ok && lane == 0) tc_commit(fin);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    // thread = one key row of the tile (TMEM lane 32*(warp%4)+lane) and 32 heads
    // (hh = warp/4 selects heads 0-31 or 32-63).
    if (threadIdx.x < kH) {  // the query's running statistics (the previous query's epilogue is done)
      m_run[threadIdx.x] = -INFINITY;
      l_run[threadIdx.x] = 0.f;
    }
    if (p.q_prep)
      prep_query(p, n, sQ, q_full, qi & 1, L.q_ready, L.hscale, L.cs_tab, abort_flag, warp, lane);
    else if (threadIdx.x < kH)
      L.hscale[threadIdx.x] = p.scale_log2;
    mbar_arrive(L.q_free);  // this thread reads Q no more (the norm reads are done)
    named_bar_sync(1, 256);
    const float* hscale = L.hscale;
    const int q4 = warp & 3, hh = warp >> 2;
    const int t = 32 * q4 + lane;
    const int h0 = 32 * hh;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    float lacc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) lacc[i] = 0.f;
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      const int T = T0 + it;
      const int b = T & 1;
      const uint32_t ph = (T >> 1) & 1;
      // S^T[b] and the tile's row flags; the TMEM load is in flight during the barrier that
      // agrees on whether both waits succeeded
      const bool got = mbar_wait(&s_full[b], ph, p.err, abort_flag) && mbar_wait(&row_ready[b], ph, p.err, abort_flag);
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + kColS + 64 * b + h0;
      uint32_t sr[32];
      tmem_ld16(s_addr, sr);
      tmem_ld16(s_addr + 16, sr + 16);
      if (named_bar_or(1, 256, !got)) {
        tmem_wait_ld();
        ok = false;
        break;
      }
      if (t == 0 && hh == 0 && it < 8) CSA_T(tslot, 40 + it);
      const bool valid = row_begin + it * kBN + t < row_end && row_ok[b * 128 + t] != 0;
      tmem_wait_ld();
      // d = logit (log2 units) - running max of its head; -inf for a row without a key
      float d[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 hs = *reinterpret_cast<const float4*>(hscale + h0 + i);
        const float4 mm = *reinterpret_cast<const float4*>(m_run + h0 + i);
        d[i] = valid ? fmaf(__uint_as_float(sr[i]), hs.x, -mm.x) : -INFINITY;
        d[i + 1] = valid ? fmaf(__uint_as_float(sr[i + 1]), hs.y, -mm.y) : -INFINITY;
        d[i + 2] = valid ? fmaf(__uint_as_float(sr[i + 2]), hs.z, -mm.z) : -INFINITY;
        d[i + 3] = valid ? fmaf(__uint_as_float(sr[i + 3]), hs.w, -mm.w) : -INFINITY;
      }
      bool over = false;
#pragma unroll
      for (int i = 0; i < 32; ++i) over |= d[i] > kRescaleThreshold;
      const bool move_max = named_bar_or(1, 256, over);  // always true on the first tile with a valid row
      if (move_max) {
        float x[32];  // the logits themselves, for the new maxima
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 hs = *reinterpret_cast<const float4*>(hscale + h0 + i);
          x[i] = valid ? __uint_as_float(sr[i]) * hs.x : -INFINITY;
          x[i + 1] = valid ? __uint_as_float(sr[i + 1]) * hs.y : -INFINITY;
          x[i + 2] = valid ? __uint_as_float(sr[i + 2]) * hs.z : -INFINITY;
          x[i + 3] = valid ? __uint_as_float(sr[i + 3]) * hs.w : -INFINITY;
        }
        xreduce32<true>(x);  // x[0] = this warp's max of head h0 + lane
        red_max[q4 * 64 + h0 + lane] = x[0];
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
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 hs = *reinterpret_cast<const float4*>(hscale + h0 + i);
          const float4 mm = *reinterpret_cast<const float4*>(m_run + h0 + i);
          d[i] = valid ? fmaf(__uint_as_float(sr[i]), hs.x, -mm.x) : -INFINITY;
          d[i + 1] = valid ? fmaf(__uint_as_float(sr[i + 1]), hs.y, -mm.y) : -INFINITY;
          d[i + 2] = valid ? fmaf(__uint_as_float(sr[i + 2]), hs.z, -mm.z) : -INFINITY;
          d[i + 3] = valid ? fmaf(__uint_as_float(sr[i + 3]), hs.w, -mm.w) : -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);  // QK of tile it + 2 may overwrite S^T[b]
      float pr[32];  // probabilities 2^d (2^-inf = 0)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        pr[i] = fast_exp2(d[i]);
        lacc[i] += pr[i];
      }
      // P[b] was last read by PV of tile it - 2, which completed before QK of this tile
      // signalled s_full (one thread issues both, and a commit covers every earlier MMA)
      // P in the third buffer, last read by PV of tile it - 1, which completed before QK of
      // this tile signalled s_full (one thread issues both; a commit covers every earlier MMA)
      uint8_t* pb = sP + 2 * 16384;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w4 = make_uint4(pack_bf16x2(pr[8 * c], pr[8 * c + 1]), pack_bf16x2(pr[8 * c + 2], pr[8 * c + 3]),
                                    pack_bf16x2(pr[8 * c + 4], pr[8 * c + 5]), pack_bf16x2(pr[8 * c + 6], pr[8 * c + 7]));
        *reinterpret_cast<uint4*>(pb + sw128(t, 4 * hh + c)) = w4;
      }
      if (move_max && it > 0) {
        // move this warp's O^T columns (heads h0..h0+31) to the new max once PV of tile
        // it - 1 is complete (PV of tile it waits for this warp's arrival on p_full)
        const bool got_o = mbar_wait(o_done, (T - 1) & 1, p.err, abort_flag);
        if (named_bar_or(1, 256, !got_o)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
      if (lane == 0) mbar_arrive(&p_full[b]);
      if (t == 0 && hh == 0 && it < 8) CSA_T(tslot, 48 + it);
    }
    // ------------------------------------------------------------ epilogue
    CSA_TB(6);
    const bool fin_ok = !named_bar_or(1, 256, !mbar_wait(fin, qi & 1, p.err, abort_flag));  // all 256 take part
    ok = ok && fin_ok;
    CSA_TB(7);
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
      for (int dp = 0; dp < 4; dp += 2) {  // two 128-dim chunks per TMEM round trip
        uint32_t o[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t ta = tmem + lane_base + kColO + 64 * (dp + c) + h0;
          tmem_ld16(ta, o[c]);
          tmem_ld16(ta + 16, o[c] + 16);
        }
        tmem_wait_ld();
        if (dp == 2) {  // O^T is read: the CTA's next query may overwrite it
          tc_fence_before();
          mbar_arrive(L.o_free);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int d = (dp + c) * 128 + t;
          if (p.splits == 1) {
            uint16_t* ob = p.out + (static_cast<size_t>(n) * kH + h0) * kD + d;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(o[c][i]) * inv_l[h0 + i]);
              ob[i * kD] = *reinterpret_cast<const uint16_t*>(&bv);
            }
          } else {
            float* pbo = p.part_o + ((static_cast<size_t>(n) * p.splits + split) * kH + h0) * kD + d;
#pragma unroll
            for (int i = 0; i < 32; ++i) pbo[i * kD] = __uint_as_float(o[c][i]);
          }
        }
      }
      if (threadIdx.x < kH) {
        const int h = threadIdx.x;
        if (p.splits == 1) {
          if (p.lse) p.lse[n * kH + h] = l_run[h] > 0.f ? (m_run[h] + log2f(l_run[h])) * 0.69314718055994531f : -INFINITY;
        } else {
          p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + h] = make_float2(m_run[h], l_run[h]);
        }
      }
    } else if (threadIdx.x < kH && p.splits > 1) {  // gave up: this split contributes nothing
      p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + threadIdx.x] = make_float2(-INFINITY, 0.f);
    }
    if (!ok) mbar_arrive(L.o_free);  // (ok is the same for all 256 threads)
  }

  if (threadIdx.x == 0) CSA_T(tslot, 3);
  CSA_TB(3);
}

// Where slab j of the K pass and slab v of the V pass go: shared-memory offset, barrier
// pair and the parity of the barrier phase (the use count of the pair, mod 2).
struct Slot2 {
  uint32_t off;
  int bar;
  uint32_t parity;
};
__device__ __forceinline__ Slot2 slot_k2(int j) {
  const int sl = j % kSlotsK2;
  Slot2 r;
  r.off = sl < kRing ? static_cast<uint32_t>(kOffRing + sl * kSlabBytes) : static_cast<uint32_t>(kOffP + (sl - kRing) * kSlabBytes);
  r.bar = sl;
  r.parity = static_cast<uint32_t>(j / kSlotsK2) & 1u;
  return r;
}

// The V pass takes the share's tiles in the order vtile(0), vtile(1), ..., a 128-dim chunk
// (two adjacent 16 KB slots) at a time.  With one or three tiles ("resident" plan), three
// chunks of the last K tile are still in the ring when the K pass ends, each in one of
// the ring's slot pairs (0,1), (2,3), (4,5) (chunks 1-3 of tile 2, chunks 0-2 of tile 0):
// that tile goes first and those chunks are not gathered again; every other chunk is
// gathered into the next slot pair of a cycle of five -- the two pairs of Q's slots
// (free after the last QK) first under the resident plan, the ring's pairs first
// otherwise.
__device__ __forceinline__ bool v_resident_plan(int n_tiles) { return n_tiles == 1 || n_tiles == 3; }
__device__ __forceinline__ int vtile(int i, int n_tiles) {
  return v_resident_plan(n_tiles) ? (i == 0 ? n_tiles - 1 : i - 1) : i;
}
// The ring pair holding chunk dc of the first V tile after the K pass, or -1 (gathered).
__device__ __forceinline__ int v_resident_pair(int dc, int n_tiles) {
  if (!v_resident_plan(n_tiles)) return -1;
  const int sl = ((n_tiles - 1) * kSlabs + 2 * dc) % kSlotsK2;  // slot_k2 of the chunk's first slab
  return (sl % 2 == 0 && sl + 1 < kRing) ? sl / 2 : -1;
}
struct VPair {
  uint32_t off;    // the first slot's offset (the second follows it)
  int bar;         // the first slot's barriers (the second: bar + 1)
  uint32_t free_parity, full_parity;
  bool q_slots;    // the pair is two of Q's slots
};
// Slots and barrier phases of the g-th gathered chunk of the V pass.  A pair's uses of
// slot_free: its K-pass uses, the resident chunk (resident plan, ring pairs), then earlier
// gathered chunks; its uses of full: the same without the resident chunk (never loaded).
__device__ __forceinline__ VPair v_pair(int g, int nK, int n_tiles) {
  const bool res = v_resident_plan(n_tiles);
  const int c = g % 5, prev = g / 5;
  const int ring = res ? c - 2 : c;  // ring pair index, or negative / >= 3 for Q's pairs
  VPair r;
  if (ring >= 0 && ring < 3) {
    const int sl = 2 * ring;
    const int k_uses = nK > sl ? (nK - 1 - sl) / kSlotsK2 + 1 : 0;  // K slabs that used this pair
    r.off = static_cast<uint32_t>(kOffRing + sl * kSlabBytes);
    r.bar = sl;
    r.free_parity = static_cast<uint32_t>(k_uses + (res ? 1 : 0) + prev) & 1u;
    r.full_parity = static_cast<uint32_t>(k_uses + prev) & 1u;
    r.q_slots = false;
  } else {
    const int q = 2 * (res ? c : c - 3);  // Q's slot pair (q, q + 1)
    r.off = static_cast<uint32_t>(kOffQ + q * kSlabBytes);
    r.bar = kRing + kPBufs + q;
    r.free_parity = r.full_parity = static_cast<uint32_t>(prev) & 1u;
    r.q_slots = true;
  }
  return r;
}

// Two-pass variant for a share of at most kMaxTiles2 tiles (decode: a query split over
// several CTAs).  The K pass is a pure stream from HBM that QK consumes as slabs land
// (S^T of tile t in TMEM columns 64 t), independent of the softmax; the softmax then runs
// once over every tile with the exact maximum (no rescaling of O^T); the V pass takes the
// rows again, tile by tile in the order vtile(), re-gathering them from L2 into slots
// that are free (or still finding them in the ring: the resident chunks of the last K
// tile), and PV accumulates O^T in columns [256, 512).  Same outputs as attend(): the normalised result or the
// unnormalised partial with its (max, sum).
__device__ __forceinline__ void attend_2pass(const AttnParams& p, const CUtensorMap& tm_q, const CUtensorMap& tm_e,
                                             const CUtensorMap& tm_w, uint8_t* smem, uint32_t tmem, int n,
                                             int split, const KeyList& kl, int row_begin, int row_end,
                                             int n_tiles) {
  const AttnSmem L(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tslot = blockIdx.x < 2 ? 4 + static_cast<int>(blockIdx.x) : -1;
  if (threadIdx.x == 0) CSA_T(tslot, 0);
  CSA_TB(2);

  if (warp >= 8 && warp < 8 + kProdWarps) {
    // ------------------------------------------------------------ gather producers
    const int pw = warp - 8;
    const int ptid = threadIdx.x - 256;
    const int my_row = gather_row(pw, lane);
    if (ptid == 0) {
      mbar_arrive_expect_tx(L.q_full, kH * kD * 2);
      for (int a = 0; a < 8; ++a) tma_load_2d(smem_u32(L.sQ + a * 8192), &tm_q, L.q_full, 128 * a, n * kH);
    }
    const int sel_here = max(0, min(row_end, kl.n_sel) - row_begin);
    const bool staged = !p.dense && sel_here <= kIdxCap;
    if (staged)
      for (int i = lane; i < sel_here; i += 32)
        if (gather_warp(i % kBN) == pw) L.sidx[i] = p.idx[static_cast<size_t>(n) * p.k + row_begin + i];
    __syncwarp();
    bool ok = true;
    const int nK = kSlabs * n_tiles;
    // K pass: tile t's slab ka is slab j = 8 t + ka of the K ring
    for (int tile = 0; ok && tile < n_tiles; ++tile) {
      const uint16_t* src_row = key_row_src(p, kl, n, row_begin + tile * kBN + my_row, row_begin, row_end,
                                            staged ? L.sidx : nullptr, true);
      const bool valid = src_row != nullptr;
      const unsigned long long src_ll = reinterpret_cast<unsigned long long>(valid ? src_row : p.entries);
      const TileBox box = tile_box(p, kl, tm_e, tm_w, row_begin + tile * kBN, row_end);
      if (ptid == 0) CSA_T(tslot, 8 + tile);
      L.row_ok[tile * 128 + my_row] = valid ? 1 : 0;  // published before the tile's first slab is issued
      mbar_arrive(&L.row_ready[tile]);
      for (int ka = 0; ka < kSlabs; ++ka) {
        const int j = tile * kSlabs + ka;
        const Slot2 sl = slot_k2(j);
        if (!warp_wait(&L.slot_free[sl.bar], sl.parity ^ 1, p.err, L.abort_flag)) {
          ok = false;
          break;
        }
        if (ptid == 0 && tslot == 4 && j < 64) CSA_T(10, j);
        gather_slab(smem_u32(smem + sl.off), box, ka, src_ll, valid, pw, lane, &L.full[sl.bar]);
      }
    }
    // V pass: the same rows again (now in L2), chunk by chunk, except the resident chunks
    bool q_free = false;  // the last QK has completed: Q's slots may take V slabs
    int g = 0;            // gathered chunks so far
    for (int vi = 0; ok && vi < n_tiles; ++vi) {
      const int tile = vtile(vi, n_tiles);
      const uint16_t* src_row = key_row_src(p, kl, n, row_begin + tile * kBN + my_row, row_begin, row_end,
                                            staged ? L.sidx : nullptr, false);
      const bool valid = src_row != nullptr;
      const unsigned long long src_ll = reinterpret_cast<unsigned long long>(valid ? src_row : p.entries);
      const TileBox box = tile_box(p, kl, tm_e, tm_w, row_begin + tile * kBN, row_end);
      if (ptid == 0) CSA_T(tslot, 8 + n_tiles + vi);
      for (int dc = 0; ok && dc < 4; ++dc) {
        if (vi == 0 && v_resident_pair(dc, n_tiles) >= 0) continue;  // still in the ring
        const VPair vp = v_pair(g++, nK, n_tiles);
        if (vp.q_slots && !q_free) {
          if (!warp_wait(&L.s_full[n_tiles - 1], 0, p.err, L.abort_flag)) {
            ok = false;
            break;
          }
          q_free = true;
        }
        for (int h = 0; h < 2; ++h) {
          if (!warp_wait(&L.slot_free[vp.bar + h], vp.free_parity ^ 1, p.err, L.abort_flag)) {
            ok = false;
            break;
          }
          gather_slab(smem_u32(smem + vp.off + h * kSlabBytes), box, 2 * dc + h, src_ll, valid, pw, lane,
                      &L.full[vp.bar + h]);
        }
      }
    }
    cp_async_wait_all();
    {
      volatile int never = 0;
      if (ptid == 0) mbar_wait(L.q_full, 0, p.err, &never);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(128, kH, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16(128, kH, true, true);
    const uint32_t base = smem_u32(smem), q0 = smem_u32(L.sQ), p0 = smem_u32(L.sP);
    const int nK = kSlabs * n_tiles;
    bool ok = warp_wait(L.q_full, 0, p.err, L.abort_flag);
    const int rope_atom = p.q_prep && p.rope_dims > 0 ? (kD - p.rope_dims) / 64 : kSlabs;
    bool q_ready_seen = rope_atom >= kSlabs;
    if (lane == 0) CSA_T(tslot, 1);
    for (int tile = 0; ok && tile < n_tiles; ++tile) {  // K pass: S^T[tile] = K Q^T
      for (int ka = 0; ka < kSlabs; ++ka) {
        const int j = tile * kSlabs + ka;
        const Slot2 sl = slot_k2(j);
        if (!warp_wait(&L.full[sl.bar], sl.parity, p.err, L.abort_flag)) {
          ok = false;
          break;
        }
        if (!q_ready_seen && ka >= rope_atom) {  // the query's rotated channels are written
          q_ready_seen = true;
          if (!warp_wait(L.q_ready, 0, p.err, L.abort_flag)) {
            ok = false;
            break;
          }
        }
        if (lane == 0 && tslot == 4 && j < 64) CSA_T(12, j);
        fence_proxy_async_smem();
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + 64 * tile, smem_desc(base + sl.off + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(q0 + ka * 8192 + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, (ka | kk) ? 1u : 0u);
          tc_commit(&L.slot_free[sl.bar]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(&L.s_full[tile]);
        CSA_T(tslot, 24 + tile);
      }
      __syncwarp();
    }
    // V pass: O^T += V^T P^T[tile], a 128-dim chunk (two adjacent slots) at a time, tiles in
    // the order vtile(0), vtile(1), ...; a tile starts as soon as its P is written (the
    // softmax publishes P tile by tile, in the same order); resident chunks need no wait
    if (lane == 0) CSA_T(tslot, 30);
    int g = 0;  // gathered chunks so far
    for (int vi = 0; ok && vi < n_tiles; ++vi) {
      const int tile = vtile(vi, n_tiles);
      if (!warp_wait(&L.row_ready[tile], 1, p.err, L.abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int dc = 0; dc < 4; ++dc) {
        const int rp = vi == 0 ? v_resident_pair(dc, n_tiles) : -1;
        uint32_t off;
        int bar;
        if (rp >= 0) {  // the K pass's slabs, still in ring slots 2 rp, 2 rp + 1
          off = static_cast<uint32_t>(kOffRing + 2 * rp * kSlabBytes);
          bar = 2 * rp;
        } else {
          const VPair vp = v_pair(g++, nK, n_tiles);
          if (!warp_wait(&L.full[vp.bar], vp.full_parity, p.err, L.abort_flag) ||
              !warp_wait(&L.full[vp.bar + 1], vp.full_parity, p.err, L.abort_flag)) {
            ok = false;
            break;
          }
          off = vp.off;
          bar = vp.bar;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + kColO2 + 64 * dc, smem_desc(base + off + ks * 2048, kSlabBytes, 1024, kSwizzle128B),
                     smem_desc(p0 + tile * 16384 + ks * 2048, 16384, 1024, kSwizzle128B), idesc_pv,
                     (vi > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&L.slot_free[bar]);
          tc_commit(&L.slot_free[bar + 1]);
        }
        __syncwarp();
      }
      if (lane == 0) CSA_T(tslot, 32 + vi);
    }
    if (ok && lane == 0) tc_commit(L.fin);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    // thread = key row t of each tile (TMEM lane 32 (warp % 4) + lane) and 32 heads
    if (p.q_prep)
      prep_query(p, n, L.sQ, L.q_full, 0, L.q_ready, L.hscale, L.cs_tab, L.abort_flag, warp, lane);
    else if (threadIdx.x < kH)
      L.hscale[threadIdx.x] = p.scale_log2;
    named_bar_sync(1, 256);
    const float* hscale = L.hscale;
    const int q4 = warp & 3, hh = warp >> 2;
    const int t = 32 * q4 + lane;
    const int h0 = 32 * hh;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q4) << 16;
    bool ok = true;
    // sweep 1: the exact maximum of every head over the CTA's rows
    float mx[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) mx[i] = -INFINITY;
    for (int it = 0; it < n_tiles; ++it) {
      const bool got = mbar_wait(&L.s_full[it], 0, p.err, L.abort_flag) &&
                       mbar_wait(&L.row_ready[it], 0, p.err, L.abort_flag);
      if (named_bar_or(1, 256, !got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (t == 0 && hh == 0) CSA_T(tslot, 40 + it);
      const bool valid = row_begin + it * kBN + t < row_end && L.row_ok[it * 128 + t] != 0;
      uint32_t sr[32];  // TMEM loads are warp-collective: every lane loads, invalid rows are masked
      const uint32_t s_addr = tmem + lane_base + 64 * it + h0;
      tmem_ld16(s_addr, sr);
      tmem_ld16(s_addr + 16, sr + 16);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 hs = *reinterpret_cast<const float4*>(hscale + h0 + i);
          mx[i] = fmaxf(mx[i], __uint_as_float(sr[i]) * hs.x);
          mx[i + 1] = fmaxf(mx[i + 1], __uint_as_float(sr[i + 1]) * hs.y);
          mx[i + 2] = fmaxf(mx[i + 2], __uint_as_float(sr[i + 2]) * hs.z);
          mx[i + 3] = fmaxf(mx[i + 3], __uint_as_float(sr[i + 3]) * hs.w);
        }
      }
    }
    if (ok) {
      xreduce32<true>(mx);  // mx[0] = this warp's max of head h0 + lane
      L.red_max[q4 * 64 + h0 + lane] = mx[0];
      named_bar_sync(1, 256);
      if (threadIdx.x < kH) {
        const int h = threadIdx.x;
        L.m_run[h] = fmaxf(fmaxf(L.red_max[h], L.red_max[64 + h]), fmaxf(L.red_max[128 + h], L.red_max[192 + h]));
      }
      named_bar_sync(1, 256);
    }
    // sweep 2: P = 2^(x - max) as bf16 per tile, and the per-thread sums, tiles in the V
    // pass's order
    float lacc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) lacc[i] = 0.f;
    for (int vi = 0; ok && vi < n_tiles; ++vi) {
      const int it = vtile(vi, n_tiles);
      const bool valid = row_begin + it * kBN + t < row_end && L.row_ok[it * 128 + t] != 0;
      float x[32];
      uint32_t sr[32];
      const uint32_t s_addr = tmem + lane_base + 64 * it + h0;
      tmem_ld16(s_addr, sr);
      tmem_ld16(s_addr + 16, sr + 16);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 mm = *reinterpret_cast<const float4*>(L.m_run + h0 + i);
          const float4 hs = *reinterpret_cast<const float4*>(hscale + h0 + i);
          x[i] = fast_exp2(fmaf(__uint_as_float(sr[i]), hs.x, -mm.x));
          x[i + 1] = fast_exp2(fmaf(__uint_as_float(sr[i + 1]), hs.y, -mm.y));
          x[i + 2] = fast_exp2(fmaf(__uint_as_float(sr[i + 2]), hs.z, -mm.z));
          x[i + 3] = fast_exp2(fmaf(__uint_as_float(sr[i + 3]), hs.w, -mm.w));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) lacc[i] += x[i];
      uint8_t* pb = L.sP + it * 16384;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w4 = make_uint4(pack_bf16x2(x[8 * c], x[8 * c + 1]), pack_bf16x2(x[8 * c + 2], x[8 * c + 3]),
                                    pack_bf16x2(x[8 * c + 4], x[8 * c + 5]), pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
        *reinterpret_cast<uint4*>(pb + sw128(t, 4 * hh + c)) = w4;
      }
      // P of this tile is complete once all 256 threads' stores are: the tile's row_ready
      // barrier, whose first phase the producers completed, takes its second phase from
      // the 8 softmax warps (128 arrivals: 16 per warp)
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane < 16) mbar_arrive(&L.row_ready[it]);
    }
    if (t == 0 && hh == 0) CSA_T(tslot, 48);
    // ------------------------------------------------------------ epilogue
    CSA_TB(6);
    const bool fin_ok = !named_bar_or(1, 256, !(ok && mbar_wait(L.fin, 0, p.err, L.abort_flag)));
    ok = ok && fin_ok;
    CSA_TB(7);
    if (t == 0 && hh == 0) CSA_T(tslot, 2);
    tc_fence_after();
    xreduce32<false>(lacc);
    L.red_sum[q4 * 64 + h0 + lane] = lacc[0];
    named_bar_sync(1, 256);
    if (threadIdx.x < kH) {
      const int h = threadIdx.x;
      L.l_run[h] = (L.red_sum[h] + L.red_sum[64 + h]) + (L.red_sum[128 + h] + L.red_sum[192 + h]);
      L.inv_l[h] = L.l_run[h] > 0.f ? 1.0f / L.l_run[h] : 0.f;
    }
    named_bar_sync(1, 256);
    if (ok) {
#pragma unroll 1
      for (int dp = 0; dp < 4; dp += 2) {
        uint32_t o[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t ta = tmem + lane_base + kColO2 + 64 * (dp + c) + h0;
          tmem_ld16(ta, o[c]);
          tmem_ld16(ta + 16, o[c] + 16);
        }
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int d = (dp + c) * 128 + t;
          if (p.splits == 1) {
            uint16_t* ob = p.out + (static_cast<size_t>(n) * kH + h0) * kD + d;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(o[c][i]) * L.inv_l[h0 + i]);
              ob[i * kD] = *reinterpret_cast<const uint16_t*>(&bv);
            }
          } else {
            float* pbo = p.part_o + ((static_cast<size_t>(n) * p.splits + split) * kH + h0) * kD + d;
#pragma unroll
            for (int i = 0; i < 32; ++i) pbo[i * kD] = __uint_as_float(o[c][i]);
          }
        }
      }
      if (threadIdx.x < kH) {
        const int h = threadIdx.x;
        const float l = L.l_run[h], m = L.m_run[h];
        if (p.splits == 1) {
          if (p.lse) p.lse[n * kH + h] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else {
          p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + h] = make_float2(l > 0.f ? m : -INFINITY, l);
        }
      }
    } else if (threadIdx.x < kH && p.splits > 1) {
      p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + threadIdx.x] = make_float2(-INFINITY, 0.f);
    }
  }
  if (threadIdx.x == 0) CSA_T(tslot, 3);
  CSA_TB(3);
}

// Barriers, running statistics and the TMEM allocation: touches no global memory, so it
// runs before the wait on the previous grid.  Returns the TMEM base address.
__device__ __forceinline__ uint32_t attn_setup(uint8_t* smem) {
  const AttnSmem L(smem);
  float* m_run = L.m_run;
  float* l_run = L.l_run;
  uint64_t* q_full = L.q_full;
  uint64_t* full = L.full;
  uint64_t* slot_free = L.slot_free;
  uint64_t* s_full = L.s_full;
  uint64_t* s_free = L.s_free;
  uint64_t* p_full = L.p_full;
  uint64_t* o_done = L.o_done;
  uint64_t* row_ready = L.row_ready;
  uint64_t* fin = L.fin;
  uint32_t* tmem_slot = L.tmem_slot;
  volatile int* abort_flag = L.abort_flag;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(L.q_ready, 256);
    mbar_init(L.q_free, 257);  // the MMA's commit after the last QK + the 256 softmax threads
    mbar_init(L.o_free, 256);
    for (int i = 0; i < kSlotBars; ++i) {
      mbar_init(&full[i], kProdThreads);
      mbar_init(&slot_free[i], 1);
    }
    for (int b = 0; b < kPBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&row_ready[b], kBN);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_free[b], 8);
      mbar_init(&p_full[b], 8);
    }
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kH) {
    m_run[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}

// The combine step of a query split S ways: heads [hb, hb + 64 / S) x 512 dims, 4 dims
// per item.  A thread's items are it = threadIdx.x + j blockDim.x; every partial of every
// item of the thread is loaded before any is used (about 20 loads from L2 in flight per
// thread instead of one round trip per item), and the per-head weights (shared memory
// wsm[hl * S + s], zero for a split that contributes nothing) are formed meanwhile.
template <int S>
__device__ __forceinline__ void merge_partials(const AttnParams& p, int n, int hb, float* wsm) {
  constexpr int kItems = kH / S * (kD / 4);
  constexpr int kPer = (kItems + kAttnThreads - 1) / kAttnThreads;  // items per thread at most
  float4 v[kPer][S];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int it = static_cast<int>(threadIdx.x) + j * kAttnThreads;
    const int hl = it / (kD / 4), d4 = it % (kD / 4);
#pragma unroll
    for (int s = 0; s < S; ++s)
      v[j][s] = it < kItems ? __ldcg(reinterpret_cast<const float4*>(
                                  p.part_o + ((static_cast<size_t>(n) * S + s) * kH + hb + hl) * kD) + d4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // while those are in flight: per head, each split's (max, sum) in one round trip, the
  // weights 2^(m_s - M) / L with L = sum_s l_s 2^(m_s - M), and the log-sum-exp
  if (static_cast<int>(threadIdx.x) < kH / S) {
    const int h = hb + static_cast<int>(threadIdx.x);
    float2 ml[S];
#pragma unroll
    for (int s = 0; s < S; ++s) ml[s] = __ldcg(&p.part_ml[(static_cast<size_t>(n) * S + s) * kH + h]);
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < S; ++s)
      if (ml[s].y > 0.f) M = fmaxf(M, ml[s].x);
    float w[S];
    float L = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
      w[s] = ml[s].y > 0.f ? exp2f(ml[s].x - M) : 0.f;
      L = fmaf(ml[s].y, w[s], L);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) wsm[threadIdx.x * S + s] = w[s] * inv;
    if (p.lse) p.lse[n * kH + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int it = static_cast<int>(threadIdx.x) + j * kAttnThreads;
    if (it >= kItems) break;
    const int hl = it / (kD / 4), d4 = it % (kD / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const float w = wsm[hl * S + s];
      if (w == 0.f) continue;  // an empty split's partial is never read as a number
      acc.x = fmaf(v[j][s].x, w, acc.x);
      acc.y = fmaf(v[j][s].y, w, acc.y);
      acc.z = fmaf(v[j][s].z, w, acc.z);
      acc.w = fmaf(v[j][s].w, w, acc.w);
    }
    const uint2 o2 = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    *reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(n) * kH + hb + hl) * kD + 4 * d4) = o2;
  }
}

// kPersist: persistent CTAs on the tile-resident pipeline (splits == 1); otherwise one query
// (or one split of a query) per CTA on either pipeline.  Two instantiations, so that each
// keeps its own register allocation.
template <bool kPersist>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_e,
                const __grid_constant__ CUtensorMap tm_w, AttnParams p) {
  CSA_TB(0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_q);
    if (p.tma_e) prefetch_tmap(&tm_e);
    if (p.tma_w) prefetch_tmap(&tm_w);
  }
  const uint32_t tmem = attn_setup(smem);
  if constexpr (kPersist) {
    // Persistent CTAs (splits == 1 on the tile-resident pipeline) take queries blockIdx.x,
    // + gridDim.x, ...: the set-up above happens once, and while the softmax warps write one
    // query's output the producers and the MMA warp already start the next.
    griddep_enter();
    CSA_TB(1);
    const AttnSmem L(smem);
    int qi = 0, T0 = 0;
    for (int n = static_cast<int>(blockIdx.x); n < p.Nq; n += static_cast<int>(gridDim.x)) {
      const KeyMeta meta = key_meta(p, n);
      if (!meta.ok) {  // a sequence out of range: no output, recorded
        if (threadIdx.x == 0) atomicExch(p.err, CSA_DEVERR_INDEX);
        continue;
      }
      const KeyList kl = key_list(p, n, meta);
      const int row_end = min(kl.win0 + kl.n_win, p.rows_per_split);
      const int n_tiles = row_end > 0 ? (row_end + kBN - 1) / kBN : 0;
      if (n_tiles == 0) {  // nothing to attend to: the softmax warps write zeros, the rest go on
        if (threadIdx.x < 256) {
          for (int i = threadIdx.x; i < kH * kD / 2; i += 256)
            reinterpret_cast<uint32_t*>(p.out + static_cast<size_t>(n) * kH * kD)[i] = 0u;
          if (p.lse && threadIdx.x < kH) p.lse[n * kH + threadIdx.x] = -INFINITY;
        }
        continue;
      }
      attend(p, tm_q, tm_e, tm_w, smem, tmem, n, 0, kl, 0, row_end, n_tiles, qi, T0);
      ++qi;
      T0 += n_tiles;
      if (*L.abort_flag) break;  // a wait gave up: every role leaves (its own waits fail at once)
    }
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  const int n = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;  // the CTA's rank in its cluster when splits > 1
  const KeyMeta meta = key_meta(p, n);      // before the wait (no kernel of this library writes it)
  griddep_enter();
  CSA_TB(1);
  const bool seq_ok = meta.ok;  // same for every CTA of the query (cluster)
  if (!seq_ok && threadIdx.x == 0 && split == 0) atomicExch(p.err, CSA_DEVERR_INDEX);
  KeyList kl{};
  int row_begin = 0, row_end = 0, n_tiles = 0;
  if (seq_ok) {
    kl = key_list(p, n, meta);
    const int nk = kl.win0 + kl.n_win;
    row_begin = split * p.rows_per_split;
    row_end = min(nk, row_begin + p.rows_per_split);
    n_tiles = row_end > row_begin ? (row_end - row_begin + kBN - 1) / kBN : 0;
  }
  if (n_tiles > 0) {
    if (p.two_pass)
      attend_2pass(p, tm_q, tm_e, tm_w, smem, tmem, n, split, kl, row_begin, row_end, n_tiles);
    else
      attend(p, tm_q, tm_e, tm_w, smem, tmem, n, split, kl, row_begin, row_end, n_tiles, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (!seq_ok) return;
  if (n_tiles == 0) {  // nothing to attend to in this split
    if (p.splits == 1) {
      for (int i = threadIdx.x; i < kH * kD / 2; i += blockDim.x)
        reinterpret_cast<uint32_t*>(p.out + static_cast<size_t>(n) * kH * kD)[i] = 0u;
      if (p.lse && threadIdx.x < kH) p.lse[n * kH + threadIdx.x] = -INFINITY;
    } else if (threadIdx.x < kH) {
      p.part_ml[(static_cast<size_t>(n) * p.splits + split) * kH + threadIdx.x] = make_float2(-INFINITY, 0.f);
    }
  }
  if (p.splits == 1) return;

  // ---------------------------------------------------------------- combine the splits
  // Every CTA of the cluster reaches this barrier (the branches above depend only on the
  // query and the split), and the release / acquire pair orders the partials in global
  // memory before the reads below.
  __threadfence();
  cluster_sync_all();
  CSA_TB(4);
  const int S = p.splits;
  const int hp = kH / S;            // heads this CTA combines
  const int hb = split * hp;
  float* wsm = reinterpret_cast<float*>(smem);  // [hp][S] weights / L
  if (S == 2) {
    merge_partials<2>(p, n, hb, wsm);
  } else if (S == 4) {
    merge_partials<4>(p, n, hb, wsm);
  } else {
    merge_partials<kMaxSplits>(p, n, hb, wsm);
  }
  CSA_TB(5);
}

int g_attn_smem[2][64];

std::atomic<int> g_batch_invariant{0};

}  // namespace

void set_batch_invariant(bool on) { g_batch_invariant.store(on ? 1 : 0); }
bool batch_invariant() { return g_batch_invariant.load() != 0; }

namespace {

// Splits of one query's key list: a power of two up to the portable cluster size, so
// that the CTAs of a query fill about one wave of SMs.  In batch-invariant mode the
// count depends on the key count alone, so a query's split boundaries, partials and
// merge order (and with them every output bit) do not depend on the batch it is in.
int split_count(int Nq, int max_keys) {
  if (batch_invariant()) {  // the fewest power-of-two splits of at most 512 rows each, up to 8
    int s = 1;
    while (s < kMaxSplits && static_cast<int64_t>(s) * 512 < max_keys) s *= 2;
    return s;
  }
  const int tiles = std::max(1, (max_keys + kBN - 1) / kBN);
  if (Nq >= kSplitSMs) return 1;
  const int want = std::min(tiles, kSplitSMs / std::max(1, Nq));
  int s = 1;
  while (s * 2 <= want && s * 2 <= kMaxSplits) s *= 2;
  return s;
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
  p.q_prep = a.q_prep;
  p.q_norm = a.q_norm;
  p.q_eps = a.q_eps;
  p.rope_dims = a.rope_dims;
  p.rope_theta = a.rope_theta;
  p.err = device_error_word();
  const int splits = split_count(a.Nq, max_keys);
  p.splits = splits;
  // One CTA per query: the tile-aligned layout, when it adds no tile at the largest key
  // list; full tiles of contiguous rows then load by TMA.  (Not in batch-invariant mode,
  // where a query's tiles, and so its rounding, must not depend on the call's sizes.)
  const int max_sel = std::min(a.dense ? a.E_max : a.k, max_keys);
  const int max_win = max_keys - max_sel;
  const int pad_keys = (max_sel + kBN - 1) / kBN * kBN + max_win;
  p.align = (splits == 1 && !batch_invariant() && (pad_keys + kBN - 1) / kBN <= (max_keys + kBN - 1) / kBN) ? 1 : 0;
  const int rows = p.align ? pad_keys : max_keys;
  p.rows_per_split = std::max(32, (((rows + splits - 1) / splits) + 31) / 32 * 32);
  p.two_pass = p.rows_per_split <= kMaxTiles2 * kBN ? 1 : 0;
  p.persist = (splits == 1 && !p.two_pass) ? 1 : 0;
  if (static_cast<int64_t>(a.Nq) * kH >= INT32_MAX) return cudaErrorInvalidValue;  // 32-bit TMA row coordinate
  CUtensorMap tm_q;  // the queries as 64-row x 128-byte boxes
  if (!encode_2d_u8(&tm_q, a.q, kD * 2, static_cast<uint64_t>(a.Nq) * kH, 128, kH, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // entry and window rows as 128-row x 128-byte boxes (one slab of a tile); a map that
  // cannot be encoded (unaligned base, too many rows for a 32-bit coordinate) leaves its
  // tiles on the gather path
  CUtensorMap tm_e{}, tm_w{};
  const auto aligned16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  const int64_t e_rows = static_cast<int64_t>(a.B) * a.E_max, w_rows = static_cast<int64_t>(a.B) * a.Tw;
  p.tma_e = (p.align && a.dense && e_rows > 0 && e_rows < INT32_MAX && aligned16(a.entries) &&
             encode_2d_u8(&tm_e, a.entries, kD * 2, static_cast<uint64_t>(e_rows), 128, kBN,
                          CU_TENSOR_MAP_SWIZZLE_128B))
                ? 1
                : 0;
  p.tma_w = (p.align && a.window != nullptr && w_rows > 0 && w_rows < INT32_MAX && aligned16(a.window) &&
             encode_2d_u8(&tm_w, a.window, kD * 2, static_cast<uint64_t>(w_rows), 128, kBN,
                          CU_TENSOR_MAP_SWIZZLE_128B))
                ? 1
                : 0;
  if (splits > 1) {
    const size_t o_bytes = static_cast<size_t>(a.Nq) * splits * kH * kD * sizeof(float);
    uintptr_t base = reinterpret_cast<uintptr_t>(a.ws);
    base = (base + 255) & ~uintptr_t(255);
    p.part_o = reinterpret_cast<float*>(base);
    p.part_ml = reinterpret_cast<float2*>(base + o_bytes);
  }
  if (p.persist) {
    cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(attn_kernel<true>), kAttnSmem, g_attn_smem[1]);
    if (e != cudaSuccess) return e;
    return launch_pdl_cluster(attn_kernel<true>, dim3(std::min(a.Nq, num_sms())), dim3(kAttnThreads), kAttnSmem, 1u, s,
                              tm_q, tm_e, tm_w, p);
  }
  cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(attn_kernel<false>), kAttnSmem, g_attn_smem[0]);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(attn_kernel<false>, dim3(a.Nq * splits), dim3(kAttnThreads), kAttnSmem,
                            static_cast<unsigned>(splits), s, tm_q, tm_e, tm_w, p);
}

}  // namespace csa
