// index.cu -- lightning indexer: block-scaled FP4 tcgen05 contraction of the query's
// indexer heads against every visible compressed key, reduced to one score per entry.
//
// Sources: "DeepSeek-V4: Million-Token Context", CSA stage (a small attention head
// scores every compressed block against the query); "Follow the white rabbit: DeepSeek
// V4's architecture in 3D", indexer paragraph (low-precision first pass adapted from
// V3.2's sparse attention); dev.to "How DeepSeek-V4 Achieves Million-Token Contexts
// ...", CSA paragraph (indexer in FP4).
//
// Score of entry j for query n:  d[h] = <q[n,h], k[j]> (MXFP4 x MXFP4, exact in
// fp32), S = fp32 chain acc = fmaf(w[n,h], max(d[h],0), acc) over h = 0..Hi-1.
//
// index_score_kernel -- one CTA per (query, share of its entry tiles): with S CTAs per
// query, CTA s takes tiles s, s + S, s + 2S, ... (the grouped and fused variants a
// contiguous run).  Entries go on the MMA M axis (128 per tile), the query's heads on N,
// the head dim on K:
//   warp 0      TMA producer: key tile 0, the query, the share's key scale bytes (a bulk
//               copy per tile), then 128 FP4 key rows (SWIZZLE_64B) per stage
//   warp 1      TMEM owner and MMA issuer: per tile, one thread tcgen05.cp's the tile's
//               scale factors into a ring of TMEM slots and issues two
//               kind::mxf4.block_scale MMAs into one of three accumulators
//   warps 2..9  first rearrange the key scale bytes into the tcgen05 scale-factor layout
//               (a tile per warp at a time), then the epilogue, two groups of four warps
//               taking alternate tiles: one thread per entry (TMEM lane), ReLU,
//               head-weighted fp32 chain, store of the score
// Barrier set-up and the TMEM allocation run before the wait on the previous grid.
//
// index_score_persistent_kernel (below) serves many queries of the common shape
// (Hi = 64, Di = 128): persistent CTAs take blocks of eight queries and load each key
// tile once per block.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>

#include "common.cuh"
#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"
#include "tmap.h"
#include "topk_regs.cuh"

namespace csa {
namespace {

constexpr int kStages = 10;         // 8 KB key stages (two CTAs per SM)
constexpr int kTileE = 128;
constexpr int kMaxTilesPerCta = 31;  // a CTA stages all of its tiles' key scale bytes in shared memory
constexpr int kIdxThreads = 320;     // producer, MMA, two epilogue groups of four warps
constexpr uint32_t kTmemCols = 256;
constexpr int kAccBufs = 3;          // accumulators of 64 columns: [0, 192)
constexpr int kSfRing = 8;           // key scale-factor slots of 4 columns: [192, 224)
constexpr uint32_t kColSFA = 64 * kAccBufs;
constexpr uint32_t kColSFB = kColSFA + 4 * kSfRing;  // 4 columns
static_assert(kColSFB + 4 <= kTmemCols, "TMEM budget (two CTAs per SM)");

struct IndexParams {
  int Nq, Hi, Di, m, B, E_max, E_stride, N;
  int tiles_per_cta, splits;
  const float* w;
  const int32_t* q_pos;
  const int32_t* q_seq;
  const int32_t* n_entries;
  const uint8_t* q_scale;
  const uint8_t* k_scale;
  const void* q_raw;  // raw queries [Nq, Hi, Di] (f32 or bf16) when kRawQ: encoded in the kernel
  int q_raw_bf16;
  float* scores;
  float* score_out;
  int32_t* err;
  int k;           // fused selection: top-k per query into idx [Nq, k] and cnt [Nq]
  int32_t* idx;
  int32_t* cnt;
};

// The fused decode variant (index_score_kernel with kFuseC > 0): a thread-block cluster of
// kFuseC CTAs per query; CTA r scores the entries [r S, (r + 1) S), S = 256 kFuseEPT, into a
// slice in its shared memory instead of global memory, then the cluster selects the query's
// top-k from those slices (topk_regs_row) -- no score round trip, one launch.  256 threads
// and ~105 KB of shared memory, so two CTAs share an SM as in the plain kernel: the producer
// (warp 0), the MMA issuer (warp 1) and one epilogue group (warps 2-5) score, and all eight
// warps select.
constexpr int kFuseThreads = 256;
constexpr int kFuseStages = 6;
// The grouped variant (kQ = 2): the two consecutive query rows of a group belong to one
// sequence (several new tokens of a sequence at decode) and share every key tile: one
// N = 128 MMA per K step scores both queries' 64 heads.  Its accumulators are 128
// columns wide, so it takes 512 TMEM columns and runs one CTA per SM (deeper key ring,
// more tiles per CTA).
constexpr int kQStages = 16;
constexpr int kQMaxTiles = 64;
template <int kFuseC, int kFuseEPT, int kQ = 1>
struct IndexShape {
  static constexpr bool kFuse = kFuseC > 0;
  static constexpr int kThreads = kFuse ? kFuseThreads : kIdxThreads;
  static constexpr int kSt = kFuse ? kFuseStages : (kQ > 1 ? kQStages : kStages);
  static constexpr int kMaxTiles = kFuse ? kFuseThreads * kFuseEPT / kTileE : (kQ > 1 ? kQMaxTiles : kMaxTilesPerCta);
  static constexpr int kRawSf = (kFuse || kQ > 1) ? 0 : kMaxTilesPerCta;  // raw scale bytes for Di = 64
  static constexpr int kSlice = kFuse ? kFuseThreads * kFuseEPT : 0;
  static constexpr uint32_t kTmem = kQ > 1 ? 512 : kTmemCols;
  static constexpr uint32_t kAccCols = 64 * kQ;                 // one accumulator: kQ x 64 heads
  static constexpr uint32_t kColSFA = kAccCols * kAccBufs;      // key scale-factor ring
  static constexpr uint32_t kColSFB = kColSFA + 4 * kSfRing;    // query scale factors (4 columns)
  static_assert(kColSFB + 4 <= kTmem, "TMEM budget");
  static constexpr int kMinBlocks = kQ > 1 ? 1 : 2;
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kSt) * 8192 + 4096 * kQ +
                                  static_cast<size_t>(kMaxTiles) * 512 + static_cast<size_t>(kRawSf) * 256 + 512 +
                                  256 * kQ + 512 + static_cast<size_t>(kSlice) * 4;
};

// kHi: number of indexer heads fixed at compile time (the head chain is straight-line
// code), or 0 to take it from p.Hi at run time.  kRawQ: the query arrives unencoded and
// the epilogue warps encode it to MXFP4 (the same rule as quantize_mxfp4_kernel) into
// the MMA's B operand and scale factors before the first tile.  kQ: queries per CTA
// sharing the key tiles (1, or 2 for the grouped variant).
template <int kHi, bool kRawQ, int kFuseC = 0, int kFuseEPT = 8, int kQ = 1>
__global__ void __launch_bounds__(IndexShape<kFuseC, kFuseEPT, kQ>::kThreads, IndexShape<kFuseC, kFuseEPT, kQ>::kMinBlocks)
    index_score_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                       IndexParams p) {
  using Shape = IndexShape<kFuseC, kFuseEPT, kQ>;
  constexpr bool kFuse = Shape::kFuse;
  static_assert(kQ == 1 || (kQ == 2 && kHi == 64 && !kRawQ && kFuseC == 0), "grouped: 64 heads, encoded queries");
  constexpr uint32_t kColSFA = Shape::kColSFA, kColSFB = Shape::kColSFB, kAccCols = Shape::kAccCols;
  constexpr int kStages = Shape::kSt;  // shadows the plain kernel's depth in this body
  // epilogue warps: two groups of four (warps 2-9); the fused kernel one (warps 2-5)
  constexpr int kEpiGroups = kFuse ? 1 : 2;
  constexpr int kEpiWarps = 4 * kEpiGroups;
  static_assert(!(kFuse && kRawQ), "the fused kernel takes pre-encoded queries");
  CSA_TB(0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // shared memory carve-up
  uint8_t* sA = smem;                                    // kStages x 8 KB (1024-aligned)
  uint8_t* sB = sA + kStages * 8192;                     // kQ x 4 KB
  uint8_t* sSF = sB + 4096 * kQ;                         // kMaxTiles x 512: key scales, scale-factor layout
  uint8_t* sSFraw = sSF + Shape::kMaxTiles * 512;        // kRawSf x 256: raw key scales when Di = 64
  uint8_t* sSFB = sSFraw + Shape::kRawSf * 256;          // 512
  float* sW = reinterpret_cast<float*>(sSFB + 512);      // [kQ][64] head weights
  float* sSlice = sW + 64 * kQ;                          // fused: this CTA's scores [kSlice]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSlice + Shape::kSlice);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* b_full = bars + 2 * kStages;
  uint64_t* sf_full = b_full + 1;    // raw key scale bytes landed
  uint64_t* sf_ready = sf_full + 1;  // epilogue warps: key scales rearranged
  uint64_t* acc_full = sf_ready + 1;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + kAccBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // Set-up that reads no global memory runs before the wait on the previous grid.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(b_full, kRawQ ? 8 : 1);
    mbar_init(sf_full, 1);
    mbar_init(sf_ready, kEpiWarps);
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Shape::kTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_enter();
  CSA_TB(1);

  // the CTA's first query row (kQ > 1: the group's), and its split of the entry tiles:
  // tiles split, split + splits, split + 2 splits, ... (the query's CTAs stream neighbouring
  // key tiles at any moment, a few windows of the cache at once rather than one stream
  // per CTA: measured faster at 128K and 1M); the fused kernel's CTA takes one contiguous
  // slice (its slice of the scores), and so does the grouped one (measured slower strided)
  constexpr bool kStrided = !kFuse && kQ == 1;
  const int q = kQ * (kFuse ? static_cast<int>(blockIdx.x) / kFuseC : static_cast<int>(blockIdx.x) / p.splits);
  const int split = kFuse ? static_cast<int>(blockIdx.x) % kFuseC : static_cast<int>(blockIdx.x) % p.splits;
  const int tiles_per_cta = kFuse ? Shape::kMaxTiles : p.tiles_per_cta;
  const int tile0 = kStrided ? split : split * tiles_per_cta;  // entry tile of local tile it: tile0 + it * tstride
  const int tstride = kStrided ? p.splits : 1;
  auto local_tiles = [&](int nv) {  // this CTA's tiles among the first ceil(nv / 128)
    const int vt = (nv + kTileE - 1) / kTileE;
    return vt > tile0 ? min((vt - 1 - tile0) / tstride + 1, tiles_per_cta) : 0;
  };
  const int seq = p.q_seq[q];
  const bool seq_ok = seq >= 0 && seq < p.B;
  if (!seq_ok && threadIdx.x == 0 && split == 0) atomicExch(p.err, CSA_DEVERR_INDEX);  // produce nothing
  const int nvis0 = seq_ok ? min(visible_entries(p.q_pos[q], p.m, p.n_entries[seq]), p.E_max) : 0;
  // grouped: the second query row, scored from the same key tiles when it names the same
  // sequence; a row naming another sequence is recorded as an error and gets -inf for
  // every entry visible to it (in this CTA's share), so that its selection is defined
  int nvis1 = 0;
  if constexpr (kQ > 1) {
    const int q1 = q + 1;
    if (q1 < p.Nq) {
      const int seq1 = p.q_seq[q1];
      const bool ok1 = seq1 >= 0 && seq1 < p.B;
      const int nv1 = ok1 ? min(visible_entries(p.q_pos[q1], p.m, p.n_entries[seq1]), p.E_max) : 0;
      if (seq_ok && seq1 == seq) {
        nvis1 = nv1;
      } else {
        if (threadIdx.x == 0 && split == 0) atomicExch(p.err, CSA_DEVERR_INDEX);
        const int n1 = local_tiles(nv1);
        for (int i = static_cast<int>(threadIdx.x); i < n1 * kTileE; i += static_cast<int>(blockDim.x)) {
          const int e = (tile0 + (i / kTileE) * tstride) * kTileE + i % kTileE;
          if (e < nv1) {
            p.scores[static_cast<size_t>(q1) * p.E_stride + e] = -INFINITY;
            if (p.score_out) p.score_out[static_cast<size_t>(q1) * p.E_max + e] = -INFINITY;
          }
        }
      }
    }
  }
  const int nvis = max(nvis0, nvis1);
  // fused: a query with at most k visible entries takes all of them (no scoring; the same
  // for every CTA of the cluster, so none reaches a cluster barrier below)
  const bool trivial = kFuse && nvis <= p.k;
  const int n_tiles = trivial ? 0 : local_tiles(nvis);  // uniform over the CTA

  const int Hi = kHi > 0 ? kHi : p.Hi;
  const int row_bytes = p.Di / 2;            // 64 (Di=128) or 32 (Di=64)
  const int a_bytes = kTileE * row_bytes;    // one stage of keys
  const int sf_row = p.Di / 32;              // scale bytes per entry: 4 or 2
  const int b_bytes = p.N * row_bytes;
  const uint32_t swz = row_bytes == 64 ? kSwizzle64B : kSwizzle32B;
  const uint32_t sbo = 8 * row_bytes;        // 8-row swizzle atom
  const int tslot = blockIdx.x < 2 ? static_cast<int>(blockIdx.x) : -1;
  if (threadIdx.x == 0) CSA_T(tslot, 0);
  CSA_TB(2);

  if (n_tiles > 0 && warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // key tile 0 first (the long pole), then the query, then every key scale byte of
      // this CTA's tiles (one bulk copy per tile, or one for a contiguous slice; they stay
      // in TMEM for the whole run), then the remaining key tiles as stages free up
      const int seq_row = seq * p.E_max;
      auto tile_e = [&](int it) { return (tile0 + it * tstride) * kTileE; };  // first entry of local tile it
      mbar_arrive_expect_tx(&full[0], a_bytes);
      CSA_T(tslot, 16);
      tma_load_2d(smem_u32(sA), &tm_k, &full[0], 0, seq_row + tile_e(0));
      if (!kRawQ) {
        mbar_arrive_expect_tx(b_full, b_bytes);
        tma_load_2d(smem_u32(sB), &tm_q, b_full, 0, q * Hi);
      }
      // entries with a scale byte in the cache: E_max and tile starts are multiples of 8,
      // so every byte count is a multiple of 16
      uint8_t* sf_dst = sf_row == 4 ? sSF : sSFraw;
      const int sf_tile = kTileE * sf_row;  // bytes of a whole tile
      if (tstride == 1) {
        const int sf_entries = min(n_tiles * kTileE, p.E_max - tile_e(0));
        const uint32_t sf_bytes = static_cast<uint32_t>(sf_entries * sf_row);
        mbar_arrive_expect_tx(sf_full, sf_bytes);
        bulk_load(smem_u32(sf_dst), p.k_scale + static_cast<size_t>(seq_row + tile_e(0)) * sf_row, sf_bytes, sf_full);
      } else {
        const int sf_entries = (n_tiles - 1) * kTileE + min(kTileE, p.E_max - tile_e(n_tiles - 1));
        mbar_arrive_expect_tx(sf_full, static_cast<uint32_t>(sf_entries * sf_row));
        for (int it = 0; it < n_tiles; ++it) {
          const uint32_t bytes = static_cast<uint32_t>(min(kTileE, p.E_max - tile_e(it)) * sf_row);
          bulk_load(smem_u32(sf_dst + it * sf_tile), p.k_scale + static_cast<size_t>(seq_row + tile_e(it)) * sf_row,
                    bytes, sf_full);
        }
      }
      for (int it = 1; it < n_tiles; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], a_bytes);
        if (it < 16) CSA_T(tslot, 16 + it);
        tma_load_2d(smem_u32(sA + st * 8192), &tm_k, &full[st], 0, seq_row + tile_e(it));
      }
    }
  } else if (n_tiles > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // scale factors of B (the query's heads) into the tcgen05 scale-factor layout:
    // row r -> byte (r % 32) * 16 + (r / 32) * 4 + block; rows >= Hi are zero (2^-127)
    if (kRawQ) {
      // the epilogue warps encoded the query into sB and sSFB
      const bool got = warp_wait(b_full, 0, p.err, abort_flag);
      if (got && lane == 0) tc_cp_32x128b_warpx4(tmem + kColSFB, smem_desc(smem_u32(sSFB), 0, 128, kSwizzleNone));
      __syncwarp();
    } else {
      uint32_t words[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;  // B row: head r % Hi of query q + r / Hi
        uint32_t v = 0;
        if (r < kQ * Hi && q + r / Hi < p.Nq) {
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
    // key scale factors of every tile, rearranged by the epilogue warps; each tile's are
    // copied into a ring of TMEM slots just before its MMAs (tcgen05 copies and MMAs of
    // one thread run in issue order, so a slot is rewritten only after the MMAs reading it)
    bool ok = warp_wait(sf_ready, 0, p.err, abort_flag);
    // one thread issues: no warp-wide polling or votes on the per-tile path
    if (ok && lane == 0) {
      ok = mbar_wait(b_full, 0, p.err, abort_flag);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int buf = it % kAccBufs;
        if (!mbar_wait(&full[st], ph, p.err, abort_flag)) break;
        if (it < 16) CSA_T(tslot, 32 + it);
        if (!mbar_wait(&acc_empty[buf], ((it / kAccBufs) & 1) ^ 1, p.err, abort_flag)) break;
        if (it < 16 && tslot == 0) CSA_T(8, it);
        tc_fence_after();
        const uint32_t sfa = tmem + kColSFA + 4 * (it % kSfRing);
        tc_cp_32x128b_warpx4(sfa, smem_desc(smem_u32(sSF + it * 512), 0, 128, kSwizzleNone));
        const uint32_t a0 = smem_u32(sA + st * 8192), b0 = smem_u32(sB);
        for (int kh = 0; kh < p.Di / 64; ++kh) {
          const uint32_t sf_id = 2 * kh;  // byte of the scale column holding blocks 2kh, 2kh+1
          mma_mxf4(tmem + kAccCols * buf, smem_desc(a0 + 32 * kh, 0, sbo, swz), smem_desc(b0 + 32 * kh, 0, sbo, swz),
                   idesc_mxf4(kTileE, p.N, sf_id, sf_id), kh > 0 ? 1u : 0u, sfa | (sf_id << 30),
                   (tmem + kColSFB) | (sf_id << 30));
        }
        tc_commit(&empty[st]);
        tc_commit(&acc_full[buf]);
        if (it < 16 && tslot == 0) CSA_T(9, it);
      }
    }
    __syncwarp();
  } else if (n_tiles > 0 && warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue (warps 2 .. 1 + kEpiWarps)
    const int ew = warp - 2;
    if (ew * 32 + lane < 64 * kQ) {  // weights of head h % 64 of query q + h / 64
      const int h = ew * 32 + lane, hq = h & 63;
      sW[h] = (hq < Hi && q + (h >> 6) < p.Nq) ? __ldg(p.w + static_cast<size_t>(q + (h >> 6)) * Hi + hq) : 0.f;
    }
    if (kRawQ) {
      // Encode the query (Hi rows x Di) into the B operand: K-major, the 16-byte chunk c of
      // row h at h * row_bytes + ((c ^ swizzle(h)) << 4) (SWIZZLE_64B: (h >> 1) & 3 for
      // 64-byte rows; SWIZZLE_32B: (h >> 2) & 1 for 32-byte rows), and its scale bytes
      // into the scale-factor layout.  Rows past Hi (N is a multiple of 16) stay zero.
      const int te = threadIdx.x - 64;  // 0..255
      for (int i = te; i < 128; i += 256) reinterpret_cast<uint32_t*>(sSFB)[i] = 0u;
      for (int i = Hi * row_bytes / 4 + te; i < p.N * row_bytes / 4; i += 256) reinterpret_cast<uint32_t*>(sB)[i] = 0u;
      named_bar_sync(1, 256);
      const int pairs = Hi * row_bytes;  // element pairs = FP4 bytes; a multiple of 16, <= 4096
      const size_t qbase = static_cast<size_t>(q) * Hi * p.Di;
      constexpr int kPer = 64 * 64 / 256;  // pairs per thread at most
      float2 xv[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {  // every load in flight before any encoding
        const int g = te + 256 * i;
        xv[i] = make_float2(0.f, 0.f);
        if (g < pairs) {
          if (p.q_raw_bf16) {
            const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q_raw) + qbase) + g);
            xv[i] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
          } else {
            xv[i] = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(p.q_raw) + qbase) + g);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int g = te + 256 * i;
        if (g - lane >= pairs) break;  // warp-uniform: whole warps past the end
        uint8_t byte, sbyte;
        mxfp4_encode_pair(xv[i].x, xv[i].y, byte, sbyte);
        if (g < pairs) {
          const int h = g / row_bytes, b = g % row_bytes;
          const int sw = row_bytes == 64 ? (h >> 1) & 3 : (h >> 2) & 1;
          sB[h * row_bytes + (((b >> 4) ^ sw) << 4) + (b & 15)] = byte;
          if ((b & 15) == 0) sSFB[(h % 32) * 16 + (h / 32) * 4 + (b >> 4)] = sbyte;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_full);
    }
    // key scales: entry-major bytes -> scale-factor layout, warp ew takes tiles ew, ew + kEpiWarps, ...
    // (word (r % 32) * 4 + r / 32 of a 512-byte slot holds the scale bytes of entry r)
    bool ok = warp_wait(sf_full, 0, p.err, abort_flag);
    if (ok) {
      for (int i = ew; i < n_tiles; i += kEpiWarps) {
        uint32_t words[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j;
          words[j] = sf_row == 4 ? *reinterpret_cast<const uint32_t*>(sSF + i * 512 + 4 * r)
                                 : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(sSFraw + i * 256 + 2 * r));
        }
        __syncwarp();
        *reinterpret_cast<uint4*>(sSF + i * 512 + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(sf_ready);
    }
    named_bar_sync(1, 32 * kEpiWarps);
    // group g (warps 2 + 4g .. 5 + 4g) takes tiles g, g + kEpiGroups, ..., so kEpiGroups tiles
    // are reduced at once; tile it sits in accumulator it % kAccBufs
    const int grp = ew >> 2;
    const int sub = warp & 3;  // TMEM lane quarter this warp may access
    for (int it = grp; ok && it < n_tiles; it += kEpiGroups) {
      const int buf = it % kAccBufs;
      if (!warp_wait(&acc_full[buf], (it / kAccBufs) & 1, p.err, abort_flag)) break;
      if (sub == 0 && lane == 0 && it < 16 && tslot == 0) CSA_T(6, it);
      tc_fence_after();
      uint32_t acc[64 * kQ];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + kAccCols * buf;
#pragma unroll
      for (int c = 0; c < 4 * kQ; ++c)
        if (16 * (c & 3) < Hi) tmem_ld16(taddr + 16 * c, acc + 16 * c);
      tmem_wait_ld();
      if (sub == 0 && lane == 0 && it < 16 && tslot == 0) CSA_T(7, it);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      const int e = (tile0 + it * tstride) * kTileE + 32 * sub + lane;
#pragma unroll
      for (int j = 0; j < kQ; ++j) {  // query q + j: columns [64 j, 64 j + Hi) of the accumulator
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < 64; h += 4) {
          if (h < Hi) {
            const float4 w4 = *reinterpret_cast<const float4*>(sW + 64 * j + h);
            s = fmaf(w4.x, fmaxf(__uint_as_float(acc[64 * j + h]), 0.f), s);
            if (h + 1 < Hi) s = fmaf(w4.y, fmaxf(__uint_as_float(acc[64 * j + h + 1]), 0.f), s);
            if (h + 2 < Hi) s = fmaf(w4.z, fmaxf(__uint_as_float(acc[64 * j + h + 2]), 0.f), s);
            if (h + 3 < Hi) s = fmaf(w4.w, fmaxf(__uint_as_float(acc[64 * j + h + 3]), 0.f), s);
          }
        }
        if (j == 0 && sub == 0 && lane == 0 && it < 16) CSA_T(tslot, 48 + it);
        if (e < (j == 0 ? nvis0 : nvis1)) {
          if constexpr (kFuse)
            sSlice[e - tile0 * kTileE] = s;
          else
            p.scores[static_cast<size_t>(q + j) * p.E_stride + e] = s;
          if (p.score_out) p.score_out[static_cast<size_t>(q + j) * p.E_max + e] = s;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) CSA_T(tslot, 1);
  CSA_TB(3);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Shape::kTmem);
  }
  if constexpr (kFuse) {
    // ---------------------------------------------------------------- selection
    if (trivial) {
      if (split == 0) {
        int32_t* out = p.idx + static_cast<size_t>(q) * p.k;
        for (int j = threadIdx.x; j < p.k; j += kFuseThreads) out[j] = j < nvis ? j : -1;
        if (threadIdx.x == 0) p.cnt[q] = nvis;
      }
      return;
    }
    // this CTA's slice (written by the epilogue warps before the barrier above) into
    // registers in the layout topk_regs_row takes: v[i] of (warp, lane) is entry
    // tile0 128 + 32 kFuseEPT warp + 32 i + lane
    using Mask = TopkMask<kFuseEPT>;
    const int e0 = tile0 * kTileE + 32 * kFuseEPT * warp + lane;
    float v[kFuseEPT];
    Mask valid = 0;
#pragma unroll
    for (int i = 0; i < kFuseEPT; ++i) {
      const bool ok = e0 + 32 * i < nvis;
      v[i] = ok ? sSlice[32 * kFuseEPT * warp + 32 * i + lane] : 0.f;
      valid |= (ok ? Mask(1) : Mask(0)) << i;
    }
    TopkParams tp{};
    tp.k = p.k;
    tp.idx = p.idx;
    tp.cnt = p.cnt;
    topk_regs_row<kFuseC, kFuseThreads, kFuseEPT>(tp, q, split, v, valid);
  }
}

// ---------------------------------------------------------------------- many queries
// index_score_persistent_kernel -- Hi = 64, Di = 128, many queries (prefill).  Queries are
// taken in blocks of eight consecutive ones.  One persistent CTA per SM deals itself
// blocks heaviest first in a zigzag over the grid (causal rows grow with position), and
// loads every key tile a block needs once for all of its queries: each tile feeds four
// N = 128 MMAs, one per pair of queries (an N = 128 block-scaled MMA costs what an N = 64
// one does), so the key stream is an eighth of one pass per query.
//   warp 0       producer: per block the eight queries' FP4 rows (TMA), scale bytes and
//                head weights (bulk copies) into one of two block buffers; per tile 128
//                FP4 key rows (TMA, SWIZZLE_64B) and their scale bytes (bulk copy)
//   warp 1       MMA: per block the pairs' scale bytes into the tcgen05 scale-factor
//                layout and TMEM; per tile the keys' (a 32 x 4 word transpose in place),
//                then per pair two kind::mxf4.block_scale MMAs (M = 128 entries, N = 128 =
//                two queries' heads, K = 64 each) into one of three accumulators
//   warps 2..25  epilogue: group g of eight warps drains accumulator g, two warps per TMEM
//                lane quarter (one per query of the pair); one thread per entry: ReLU,
//                head-weighted fp32 chain, store
// A block whose queries span several sequences runs as segments, one per sequence run,
// each with its own key tiles; the pairs a segment touches compute both halves and keep
// the segment's queries.  The producer writes each block's query information (validity,
// visible counts, segments) into shared memory beside the block buffer, published by the
// buffer's barrier, so every role follows the same (segment, tile, pair) order; a block
// without a valid query still passes through the buffer protocol.  Every wait sleeps
// (try_wait with a suspend-time hint) instead of polling: 26 warps polling mbarriers
// took shared-memory bandwidth from the warps doing the work.
constexpr int kPStages = 10;
constexpr int kBlkQ = 8;               // queries per block
constexpr int kPairs = kBlkQ / 2;      // N = 128 MMAs per key tile
constexpr int kPAcc = 3;               // accumulators of 128 columns
constexpr int kPGroups = kPAcc;        // epilogue group g drains accumulator g
constexpr int kPEpiWarps = 8;          // per group: 4 lane quarters x 2 queries
constexpr int kPThreads = 32 * (2 + kPEpiWarps * kPGroups);
constexpr uint32_t kPTmemCols = 512;
constexpr uint32_t kPColSFA = 128 * kPAcc;              // ring of kSfRing x 4 columns
constexpr uint32_t kPColSFB = kPColSFA + 4 * kSfRing;   // 2 blocks x kPairs x 4 columns
static_assert(kPColSFB + 2 * kPairs * 4 <= kPTmemCols, "TMEM budget (one CTA per SM)");

// The eight queries of block b: validity, sequence, visible entries, and the segments
// (maximal runs of valid queries sharing a sequence, in query order).
struct BlockInfo {
  int nseg;
  int seq[kBlkQ], nvis[kBlkQ];
  uint32_t valid;            // bit g: query 8b + g exists and has a sequence in range
  int seg_seq[kBlkQ], seg_lo[kBlkQ], seg_hi[kBlkQ], seg_nt[kBlkQ];
};

__device__ __forceinline__ void block_info(const IndexParams& p, int b, BlockInfo& bi) {
  bi.valid = 0;
  bi.nseg = 0;
#pragma unroll
  for (int g = 0; g < kBlkQ; ++g) {
    const int q = b * kBlkQ + g;
    bi.seq[g] = -1;
    bi.nvis[g] = 0;
    if (q < p.Nq) {
      const int s = p.q_seq[q];
      if (s >= 0 && s < p.B) {
        bi.seq[g] = s;
        bi.nvis[g] = min(visible_entries(p.q_pos[q], p.m, p.n_entries[s]), p.E_max);
        bi.valid |= 1u << g;
      }
    }
  }
  for (int g = 0; g < kBlkQ; ++g) {
    if (!(bi.valid >> g & 1u)) continue;
    const int nt = (bi.nvis[g] + kTileE - 1) / kTileE;
    if (bi.nseg > 0 && bi.seg_seq[bi.nseg - 1] == bi.seq[g]) {
      bi.seg_hi[bi.nseg - 1] = g;
      bi.seg_nt[bi.nseg - 1] = max(bi.seg_nt[bi.nseg - 1], nt);
    } else {
      bi.seg_seq[bi.nseg] = bi.seq[g];
      bi.seg_lo[bi.nseg] = g;
      bi.seg_hi[bi.nseg] = g;
      bi.seg_nt[bi.nseg] = nt;
      ++bi.nseg;
    }
  }
}

struct PersistSmem {
  uint8_t* sA;     // kPStages x 8 KB key tiles (1024-aligned)
  uint8_t* sSFA;   // kPStages x 512: a tile's scale bytes (raw, then scale-factor layout)
  uint8_t* sB;     // 2 x kBlkQ x 4 KB query rows (1024-aligned); pair p = 8 KB at 8 KB p
  uint8_t* sSFB;   // 2 x kBlkQ x 256 raw scale bytes; pair p's 512 B become its layout
  float* sW;       // 2 x kBlkQ x 64 head weights
  BlockInfo* info; // 2: the block in each buffer, written by the producer
  uint64_t* full;       // [kPStages]
  uint64_t* empty;      // [kPStages]
  uint64_t* blk_full;   // [2]
  uint64_t* blk_empty;  // [2]
  uint64_t* acc_full;   // [kPAcc]
  uint64_t* acc_empty;  // [kPAcc]
  uint64_t* fin;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  __device__ explicit PersistSmem(uint8_t* s) {
    sA = s;
    sSFA = sA + kPStages * 8192;
    sB = sSFA + kPStages * 512;
    sSFB = sB + 2 * kBlkQ * 4096;
    sW = reinterpret_cast<float*>(sSFB + 2 * kBlkQ * 256);
    info = reinterpret_cast<BlockInfo*>(sW + 2 * kBlkQ * 64);
    full = reinterpret_cast<uint64_t*>(info + 2);
    empty = full + kPStages;
    blk_full = empty + kPStages;
    blk_empty = blk_full + 2;
    acc_full = blk_empty + 2;
    acc_empty = acc_full + kPAcc;
    fin = acc_empty + kPAcc;
    tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  }
};
constexpr size_t kPersistSmem = 1024 + kPStages * (8192 + 512) + 2 * kBlkQ * (4096 + 256 + 256) +
                                2 * sizeof(BlockInfo) + 8 * (2 * kPStages + 4 + 2 * kPAcc + 1) + 16;
static_assert(sizeof(BlockInfo) % 8 == 0, "barriers after the block infos stay 8-byte aligned");
static_assert(kPersistSmem <= 227 * 1024, "shared memory budget");

// block dealt to this CTA in round r (zigzag over the grid, heaviest blocks first), or -1
__device__ __forceinline__ int dealt_block(int r, int nblk) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int k = r * G + ((r & 1) ? (G - 1 - c) : c);
  return k < nblk ? nblk - 1 - k : -1;
}

// In place: 128 words of row-major scale bytes (word r = the 4 scale bytes of row r) ->
// the scale-factor layout of a 32x128b copy (word 4 (r % 32) + r / 32).  Rows at or past
// `rows` are zero.  All 32 lanes of the warp call it.
__device__ __forceinline__ void sf_transpose(uint8_t* buf, int rows, int lane) {
  uint32_t* w = reinterpret_cast<uint32_t*>(buf);
  uint32_t v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = lane + 32 * i < rows ? w[lane + 32 * i] : 0u;
  __syncwarp();
  reinterpret_cast<uint4*>(buf)[lane] = make_uint4(v[0], v[1], v[2], v[3]);
}

__global__ void __launch_bounds__(kPThreads, 1)
    index_score_persistent_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                                  IndexParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const PersistSmem L(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kHiP = 64;
  constexpr uint32_t kSbo = 8 * 64;  // 8-row SWIZZLE_64B atom of 64-byte rows
  const int nblk = (p.Nq + kBlkQ - 1) / kBlkQ;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&L.full[s], 1);
      mbar_init(&L.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&L.blk_full[b], 1);
      mbar_init(&L.blk_empty[b], 1 + kPEpiWarps * kPGroups);  // the MMA thread's commit, then each epilogue warp
    }
    for (int i = 0; i < kPAcc; ++i) {
      mbar_init(&L.acc_full[i], 1);
      mbar_init(&L.acc_empty[i], kPEpiWarps);
    }
    mbar_init(L.fin, 1);
    *L.abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(L.tmem_slot, kPTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *L.tmem_slot;
  griddep_enter();
  volatile int* abort_flag = L.abort_flag;
  const bool stamp = blockIdx.x == 0;  // development timing builds: CTA 0's pipeline events
  if (stamp && threadIdx.x == 0) CSA_T(9, 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int T = 0;
      BlockInfo bi;
      for (int r = 0; ok; ++r) {  // blocks alternate between the two buffers, empty ones too
        const int b = dealt_block(r, nblk);
        if (b < 0) break;
        block_info(p, b, bi);
        for (int g = 0; g < kBlkQ; ++g)  // sequence ids out of range produce nothing
          if (b * kBlkQ + g < p.Nq && !(bi.valid >> g & 1u)) atomicExch(p.err, CSA_DEVERR_INDEX);
        const int bb = r & 1;
        if (!mbar_wait(&L.blk_empty[bb], ((r >> 1) & 1) ^ 1, p.err, abort_flag)) break;
        if (stamp && r < 64) CSA_T(15, r);
        L.info[bb] = bi;  // published by the arrival below
        mbar_arrive_expect_tx(&L.blk_full[bb], __popc(bi.valid) * (4096 + 256 + 256));
        for (int g = 0; g < kBlkQ; ++g) {
          if (!(bi.valid >> g & 1u)) continue;
          const int q = b * kBlkQ + g;
          const int slot = bb * kBlkQ + g;
          tma_load_2d(smem_u32(L.sB + slot * 4096), &tm_q, &L.blk_full[bb], 0, q * kHiP);
          bulk_load(smem_u32(L.sSFB + slot * 256), p.q_scale + static_cast<size_t>(q) * kHiP * 4, 256, &L.blk_full[bb]);
          bulk_load(smem_u32(L.sW + slot * 64), p.w + static_cast<size_t>(q) * kHiP, 256, &L.blk_full[bb]);
        }
        for (int sg = 0; ok && sg < bi.nseg; ++sg) {
          for (int j = 0; j < bi.seg_nt[sg]; ++j, ++T) {
            const int st = T % kPStages;
            if (!mbar_wait(&L.empty[st], ((T / kPStages) & 1) ^ 1, p.err, abort_flag)) {
              ok = false;
              break;
            }
            const int e0 = j * kTileE;
            const int row0 = bi.seg_seq[sg] * p.E_max + e0;
            // scale bytes of the entries the cache holds (E_max and e0 are multiples of 8)
            const uint32_t sf_bytes = static_cast<uint32_t>(min(kTileE, p.E_max - e0) * 4);
            if (stamp && T < 64) CSA_T(10, T);
            mbar_arrive_expect_tx(&L.full[st], 8192 + sf_bytes);
            tma_load_2d(smem_u32(L.sA + st * 8192), &tm_k, &L.full[st], 0, row0);
            bulk_load(smem_u32(L.sSFA + st * 512), p.k_scale + static_cast<size_t>(row0) * 4, sf_bytes, &L.full[st]);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    bool ok = true;
    int T = 0, U = 0;
    for (int r = 0; ok; ++r) {
      if (dealt_block(r, nblk) < 0) break;
      const int bb = r & 1;
      ok = warp_wait_sleep(&L.blk_full[bb], (r >> 1) & 1, p.err, abort_flag);
      if (!ok) break;
      const BlockInfo& bi = L.info[bb];
      if (bi.nseg == 0) {
        if (lane == 0) mbar_arrive(&L.blk_empty[bb]);
        __syncwarp();
        continue;
      }
      if (stamp && lane == 0 && r < 64) CSA_T(16, r);
#pragma unroll 1
      for (int pr = 0; pr < kPairs; ++pr) sf_transpose(L.sSFB + (bb * kBlkQ + 2 * pr) * 256, 128, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
        for (int pr = 0; pr < kPairs; ++pr)
          tc_cp_32x128b_warpx4(tmem + kPColSFB + 4 * (bb * kPairs + pr),
                               smem_desc(smem_u32(L.sSFB + (bb * kBlkQ + 2 * pr) * 256), 0, 128, kSwizzleNone));
      }
      __syncwarp();
      for (int sg = 0; ok && sg < bi.nseg; ++sg) {
        const int p_lo = bi.seg_lo[sg] >> 1, p_hi = bi.seg_hi[sg] >> 1;
        for (int j = 0; ok && j < bi.seg_nt[sg]; ++j, ++T) {
          const int st = T % kPStages;
          ok = warp_wait_sleep(&L.full[st], (T / kPStages) & 1, p.err, abort_flag);
          if (!ok) break;
          if (stamp && lane == 0 && T < 64) CSA_T(11, T);
          sf_transpose(L.sSFA + st * 512, min(kTileE, p.E_max - j * kTileE), lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc_fence_after();
            const uint32_t sfa = tmem + kPColSFA + 4 * (T % kSfRing);
            tc_cp_32x128b_warpx4(sfa, smem_desc(smem_u32(L.sSFA + st * 512), 0, 128, kSwizzleNone));
            const uint32_t a0 = smem_u32(L.sA + st * 8192);
            for (int pr = p_lo; ok && pr <= p_hi; ++pr, ++U) {
              const int buf = U % kPAcc;
              ok = mbar_wait_sleep(&L.acc_empty[buf], ((U / kPAcc) & 1) ^ 1, p.err, abort_flag);
              if (!ok) break;
              tc_fence_after();
              const uint32_t b0 = smem_u32(L.sB + (bb * kBlkQ + 2 * pr) * 4096);
              const uint32_t sfb = tmem + kPColSFB + 4 * (bb * kPairs + pr);
#pragma unroll
              for (int kh = 0; kh < 2; ++kh) {
                const uint32_t sf_id = 2 * kh;  // byte of the scale column holding blocks 2kh, 2kh+1
                mma_mxf4(tmem + 128 * buf, smem_desc(a0 + 32 * kh, 0, kSbo, kSwizzle64B),
                         smem_desc(b0 + 32 * kh, 0, kSbo, kSwizzle64B), idesc_mxf4(kTileE, 2 * kHiP, sf_id, sf_id),
                         kh > 0 ? 1u : 0u, sfa | (sf_id << 30), sfb | (sf_id << 30));
              }
              tc_commit(&L.acc_full[buf]);
            }
            tc_commit(&L.empty[st]);  // the key tile's last MMA has read it
            if (stamp && T < 64) CSA_T(12, T);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          U = __shfl_sync(0xffffffffu, U, 0);
        }
      }
      if (lane == 0 && ok) tc_commit(&L.blk_empty[bb]);  // the block's MMAs no longer read its buffer
      __syncwarp();
    }
    if (lane == 0) {  // every tcgen05 operation of this thread (and its commits) has completed
      tc_commit(L.fin);
      volatile int never = 0;
      mbar_wait(L.fin, 0, p.err, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..25)
    const int grp = (warp - 2) / kPEpiWarps;  // accumulator this group drains
    const int half = ((warp - 2) % kPEpiWarps) >> 2;  // query of the pair: 2 pr + half
    const int sub = warp & 3;                 // TMEM lane quarter this warp may access
    const uint32_t lane_base = static_cast<uint32_t>(32 * sub) << 16;
    bool ok = true;
    int U = 0;
    for (int r = 0; ok; ++r) {
      const int b = dealt_block(r, nblk);
      if (b < 0) break;
      const int bb = r & 1;
      ok = warp_wait_sleep(&L.blk_full[bb], (r >> 1) & 1, p.err, abort_flag);  // the block and its head weights
      const BlockInfo& bi = L.info[bb];
      for (int sg = 0; ok && sg < bi.nseg; ++sg) {
        const int p_lo = bi.seg_lo[sg] >> 1, p_hi = bi.seg_hi[sg] >> 1;
        const int s_seq = bi.seg_seq[sg];
        for (int j = 0; ok && j < bi.seg_nt[sg]; ++j) {
          for (int pr = p_lo; ok && pr <= p_hi; ++pr, ++U) {
            if (U % kPAcc != grp) continue;
            ok = warp_wait_sleep(&L.acc_full[grp], (U / kPAcc) & 1, p.err, abort_flag);
            if (!ok) break;
            if (stamp && sub == 0 && half == 0 && lane == 0 && U < 64) CSA_T(13, U);
            tc_fence_after();
            const int g = 2 * pr + half;
            const bool keep = (bi.valid >> g & 1u) && bi.seq[g] == s_seq && g >= bi.seg_lo[sg] && g <= bi.seg_hi[sg];
            const float* w = L.sW + (bb * kBlkQ + g) * 64;
            const uint32_t taddr = tmem + lane_base + 128 * grp + 64 * half;
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // 32 heads per TMEM read
              uint32_t x[32];
              tmem_ld16(taddr + 32 * c, x);
              tmem_ld16(taddr + 32 * c + 16, x + 16);
              tmem_wait_ld();
              if (c == 1) {  // the accumulator is read: the next MMA may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&L.acc_empty[grp]);
              }
#pragma unroll
              for (int hh = 0; hh < 32; hh += 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(w + 32 * c + hh);
                s = fmaf(w4.x, fmaxf(__uint_as_float(x[hh]), 0.f), s);
                s = fmaf(w4.y, fmaxf(__uint_as_float(x[hh + 1]), 0.f), s);
                s = fmaf(w4.z, fmaxf(__uint_as_float(x[hh + 2]), 0.f), s);
                s = fmaf(w4.w, fmaxf(__uint_as_float(x[hh + 3]), 0.f), s);
              }
            }
            const int e = j * kTileE + 32 * sub + lane;
            if (keep && e < bi.nvis[g]) {
              const int q = b * kBlkQ + g;
              p.scores[static_cast<size_t>(q) * p.E_stride + e] = s;
              if (p.score_out) p.score_out[static_cast<size_t>(q) * p.E_max + e] = s;
            }
            if (stamp && sub == 0 && half == 0 && lane == 0 && U < 64) CSA_T(14, U);
          }
        }
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&L.blk_empty[bb]);  // done with the block's weights
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPTmemCols);
  }
}

int g_index_smem[6][64];

}  // namespace

size_t index_workspace_bytes(int Nq, int E_max, int /*k*/) {
  const size_t stride = (static_cast<size_t>(E_max) + 3) & ~size_t(3);
  return static_cast<size_t>(Nq) * stride * sizeof(float) + 256;
}

cudaError_t launch_index_score(const IndexArgs& a, cudaStream_t s) {
  const int row_bytes = a.Di / 2;
  const bool grouped = a.q_group == 2;
  if (grouped && (a.Hi != 64 || a.Di != 128 || a.q_raw != nullptr)) return cudaErrorInvalidValue;
  const int N = grouped ? 128 : std::max(16, (a.Hi + 15) / 16 * 16);  // B rows: one query's heads, or a pair's
  CUtensorMap tm_k, tm_q;
  const CUtensorMapSwizzle swz = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!encode_2d_u8(&tm_k, a.k_fp4, row_bytes, static_cast<uint64_t>(a.B) * a.E_max, row_bytes, kTileE, swz))
    return cudaErrorInvalidValue;
  // raw queries are encoded in the kernel: the query map is then unused (any valid map)
  if (!(a.q_raw != nullptr
            ? encode_2d_u8(&tm_q, a.k_fp4, row_bytes, static_cast<uint64_t>(a.B) * a.E_max, row_bytes, N, swz)
            : encode_2d_u8(&tm_q, a.q_fp4, row_bytes, static_cast<uint64_t>(a.Nq) * a.Hi, row_bytes, N, swz)))
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
  // splits of each query's (group's) entry range: about one wave of CTAs, and no CTA
  // with more tiles than it stages scale bytes for
  const int units = grouped ? (a.Nq + 1) / 2 : a.Nq;
  const int per_sm = grouped ? 1 : 2;
  const int max_tiles = grouped ? kQMaxTiles : kMaxTilesPerCta;
  int splits = std::max(1, std::min(tiles_max, per_sm * num_sms() / std::max(1, units)));
  splits = std::max(splits, (tiles_max + max_tiles - 1) / max_tiles);
  p.tiles_per_cta = (tiles_max + splits - 1) / splits;
  p.splits = (tiles_max + p.tiles_per_cta - 1) / p.tiles_per_cta;
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.q_seq = a.q_seq;
  p.n_entries = a.n_entries;
  p.q_scale = a.q_scale;
  p.k_scale = a.k_scale;
  p.scores = a.scores_ws;
  p.score_out = a.score_out;
  p.err = device_error_word();

  if (grouped) {  // pairs of queries of one sequence share every key tile
    constexpr size_t smem = IndexShape<0, 8, 2>::kSmem;
    const cudaError_t e =
        set_dyn_smem(reinterpret_cast<const void*>(index_score_kernel<64, false, 0, 8, 2>), smem, g_index_smem[5]);
    if (e != cudaSuccess) return e;
    return launch_pdl(index_score_kernel<64, false, 0, 8, 2>, dim3(units * p.splits), dim3(kIdxThreads), smem, s,
                      tm_k, tm_q, p);
  }

  // many pre-encoded queries of the common shape: persistent CTAs, several queries each
  if (a.q_raw == nullptr && a.Hi == 64 && a.Di == 128 && a.Nq >= 2 * num_sms() &&
      (reinterpret_cast<uintptr_t>(a.w) & 15u) == 0 && (reinterpret_cast<uintptr_t>(a.q_scale) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(a.k_scale) & 15u) == 0) {
    const cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(index_score_persistent_kernel), kPersistSmem,
                                       g_index_smem[4]);
    if (e != cudaSuccess) return e;
    const int nblk = (a.Nq + kBlkQ - 1) / kBlkQ;
    return launch_pdl(index_score_persistent_kernel, dim3(std::min(nblk, num_sms())), dim3(kPThreads), kPersistSmem,
                      s, tm_k, tm_q, p);
  }

  const size_t smem = IndexShape<0, 8>::kSmem;
  p.q_raw = a.q_raw;
  p.q_raw_bf16 = a.q_raw_bf16;
  const dim3 grid(a.Nq * p.splits), block(kIdxThreads);
  auto go = [&](auto kern, int slot) -> cudaError_t {
    const cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(kern), smem, g_index_smem[slot]);
    return e != cudaSuccess ? e : launch_pdl(kern, grid, block, smem, s, tm_k, tm_q, p);
  };
  if (a.q_raw != nullptr)
    return a.Hi == 64 ? go(index_score_kernel<64, true>, 2) : go(index_score_kernel<0, true>, 3);
  return a.Hi == 64 ? go(index_score_kernel<64, false>, 0) : go(index_score_kernel<0, false>, 1);
}

namespace {
int g_fuse_smem[6][64];

template <int C, int EPT>
cudaError_t launch_fused_t(const CUtensorMap& tm_k, const CUtensorMap& tm_q, const IndexParams& p, int Nq,
                           cudaStream_t s, int slot) {
  auto kern = index_score_kernel<64, false, C, EPT>;
  constexpr size_t smem = IndexShape<C, EPT>::kSmem;
  const cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(kern), smem, g_fuse_smem[slot]);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(kern, dim3(Nq * C), dim3(kFuseThreads), smem, static_cast<unsigned>(C), s, tm_k, tm_q, p);
}
}  // namespace

namespace {
std::atomic<int> g_index_fusion{0};
}  // namespace

void set_index_fusion(bool on) { g_index_fusion.store(on ? 1 : 0); }

bool index_topk_fusable(int Nq, int Hi, int Di, int E_max, int k, bool raw_q, int* C_out, int* ept_out) {
  if (g_index_fusion.load() == 0) return false;
  if (raw_q || Hi != 64 || Di != 128 || k < 1 || Nq < 1) return false;
  // the largest cluster for which two CTAs per SM hold every query and the slices hold the
  // row; the fused kernel only pays when the CTAs are at least one per SM
  const int sms = num_sms();
  int C = 0;
  for (int c = 8; c >= 2 && C == 0; c >>= 1)
    if (static_cast<int64_t>(Nq) * c <= 2 * sms && static_cast<int64_t>(c) * kFuseThreads * 16 >= E_max) C = c;
  if (C == 0 || static_cast<int64_t>(Nq) * C < sms) return false;
  if (C_out) *C_out = C;
  if (ept_out) *ept_out = static_cast<int64_t>(C) * kFuseThreads * 8 >= E_max ? 8 : 16;
  return true;
}

cudaError_t launch_index_topk_fused(const IndexArgs& a, cudaStream_t s, bool* launched) {
  *launched = false;
  int C = 0, ept = 0;
  if (a.idx_out == nullptr || a.cnt_out == nullptr || a.q_group == 2 ||
      !index_topk_fusable(a.Nq, a.Hi, a.Di, a.E_max, a.k, a.q_raw != nullptr, &C, &ept))
    return cudaSuccess;
  CUtensorMap tm_k, tm_q;
  if (!encode_2d_u8(&tm_k, a.k_fp4, 64, static_cast<uint64_t>(a.B) * a.E_max, 64, kTileE, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_2d_u8(&tm_q, a.q_fp4, 64, static_cast<uint64_t>(a.Nq) * a.Hi, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  IndexParams p{};
  p.Nq = a.Nq;
  p.Hi = a.Hi;
  p.Di = a.Di;
  p.m = a.m;
  p.B = a.B;
  p.E_max = a.E_max;
  p.E_stride = a.E_stride;
  p.N = 64;
  p.tiles_per_cta = kFuseThreads * ept / kTileE;
  p.splits = C;
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.q_seq = a.q_seq;
  p.n_entries = a.n_entries;
  p.q_scale = a.q_scale;
  p.k_scale = a.k_scale;
  p.scores = nullptr;
  p.score_out = a.score_out;
  p.err = device_error_word();
  p.k = a.k;
  p.idx = a.idx_out;
  p.cnt = a.cnt_out;
  cudaError_t e;
  if (C == 8)
    e = ept == 8 ? launch_fused_t<8, 8>(tm_k, tm_q, p, a.Nq, s, 0) : launch_fused_t<8, 16>(tm_k, tm_q, p, a.Nq, s, 1);
  else if (C == 4)
    e = ept == 8 ? launch_fused_t<4, 8>(tm_k, tm_q, p, a.Nq, s, 2) : launch_fused_t<4, 16>(tm_k, tm_q, p, a.Nq, s, 3);
  else
    e = ept == 8 ? launch_fused_t<2, 8>(tm_k, tm_q, p, a.Nq, s, 4) : launch_fused_t<2, 16>(tm_k, tm_q, p, a.Nq, s, 5);
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace csa
