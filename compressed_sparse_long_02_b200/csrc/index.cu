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
// index_score_kernel -- one CTA per (query, run of entry tiles).  Entries go on the
// MMA M axis (128 per tile), the query's heads on N, the head dim on K:
//   warp 0      TMA producer: key tile 0, the query, the run's key scale bytes (one bulk
//               copy), then 128 FP4 key rows (SWIZZLE_64B) per stage
//   warp 1      TMEM owner and MMA issuer: per tile, one thread tcgen05.cp's the tile's
//               scale factors into a ring of TMEM slots and issues two
//               kind::mxf4.block_scale MMAs into one of three accumulators
//   warps 2..9  first rearrange the key scale bytes into the tcgen05 scale-factor layout
//               (a tile per warp at a time), then the epilogue, two groups of four warps
//               taking alternate tiles: one thread per entry (TMEM lane), ReLU,
//               head-weighted fp32 chain, store of the score
// Barrier set-up and the TMEM allocation run before the wait on the previous grid.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "internal.h"
#include "mxfp4.cuh"
#include "ptx.cuh"
#include "tmap.h"

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
};

// kHi: number of indexer heads fixed at compile time (the head chain is straight-line
// code), or 0 to take it from p.Hi at run time.  kRawQ: the query arrives unencoded and
// the epilogue warps encode it to MXFP4 (the same rule as quantize_mxfp4_kernel) into
// the MMA's B operand and scale factors before the first tile.
template <int kHi, bool kRawQ>
__global__ void __launch_bounds__(kIdxThreads, 2)
    index_score_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                       IndexParams p) {
  CSA_TB(0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // shared memory carve-up
  uint8_t* sA = smem;                                    // kStages x 8 KB (1024-aligned)
  uint8_t* sB = sA + kStages * 8192;                     // 4 KB
  uint8_t* sSF = sB + 4096;                              // kMaxTilesPerCta x 512: key scales, scale-factor layout
  uint8_t* sSFraw = sSF + kMaxTilesPerCta * 512;         // kMaxTilesPerCta x 256: raw key scales when Di = 64
  uint8_t* sSFB = sSFraw + kMaxTilesPerCta * 256;        // 512
  float* sW = reinterpret_cast<float*>(sSFB + 512);      // [64] head weights
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + 64);
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
    mbar_init(sf_ready, 8);
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
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_enter();
  CSA_TB(1);

  const int q = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int seq = p.q_seq[q];
  const bool seq_ok = seq >= 0 && seq < p.B;
  if (!seq_ok && threadIdx.x == 0 && split == 0) atomicExch(p.err, CSA_DEVERR_INDEX);  // produce nothing
  const int nvis = seq_ok ? min(visible_entries(p.q_pos[q], p.m, p.n_entries[seq]), p.E_max) : 0;
  const int t_begin = split * p.tiles_per_cta;
  const int t_end = min((nvis + kTileE - 1) / kTileE, t_begin + p.tiles_per_cta);
  const int n_tiles = t_end - t_begin;  // uniform over the CTA

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
      // this CTA's tiles in one bulk copy (they stay in TMEM for the whole run), then the
      // remaining key tiles as stages free up
      const int row0 = seq * p.E_max + t_begin * kTileE;
      mbar_arrive_expect_tx(&full[0], a_bytes);
      CSA_T(tslot, 16);
      tma_load_2d(smem_u32(sA), &tm_k, &full[0], 0, row0);
      if (!kRawQ) {
        mbar_arrive_expect_tx(b_full, b_bytes);
        tma_load_2d(smem_u32(sB), &tm_q, b_full, 0, q * Hi);
      }
      // entries with a scale byte in the cache: E_max and tile starts are multiples of 8,
      // so the byte count is a multiple of 16
      const int sf_entries = min(n_tiles * kTileE, p.E_max - t_begin * kTileE);
      const uint32_t sf_bytes = static_cast<uint32_t>(sf_entries * sf_row);
      mbar_arrive_expect_tx(sf_full, sf_bytes);
      bulk_load(smem_u32(sf_row == 4 ? sSF : sSFraw), p.k_scale + static_cast<size_t>(row0) * sf_row, sf_bytes,
                sf_full);
      for (int it = 1; it < n_tiles; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], a_bytes);
        if (it < 16) CSA_T(tslot, 16 + it);
        tma_load_2d(smem_u32(sA + st * 8192), &tm_k, &full[st], 0, row0 + it * kTileE);
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
          mma_mxf4(tmem + 64 * buf, smem_desc(a0 + 32 * kh, 0, sbo, swz), smem_desc(b0 + 32 * kh, 0, sbo, swz),
                   idesc_mxf4(kTileE, p.N, sf_id, sf_id), kh > 0 ? 1u : 0u, sfa | (sf_id << 30),
                   (tmem + kColSFB) | (sf_id << 30));
        }
        tc_commit(&empty[st]);
        tc_commit(&acc_full[buf]);
        if (it < 16 && tslot == 0) CSA_T(9, it);
      }
    }
    __syncwarp();
  } else if (n_tiles > 0) {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int ew = warp - 2;
    if (ew * 32 + lane < 64) {
      const int h = ew * 32 + lane;
      sW[h] = h < Hi ? __ldg(p.w + static_cast<size_t>(q) * Hi + h) : 0.f;
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
    // key scales: entry-major bytes -> scale-factor layout, warp ew takes tiles ew, ew + 8, ...
    // (word (r % 32) * 4 + r / 32 of a 512-byte slot holds the scale bytes of entry r)
    bool ok = warp_wait(sf_full, 0, p.err, abort_flag);
    if (ok) {
      for (int i = ew; i < n_tiles; i += 8) {
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
    named_bar_sync(1, 256);
    // group 0 (warps 2-5) takes even tiles, group 1 (warps 6-9) odd tiles, so two tiles
    // are reduced at once; tile it sits in accumulator it % kAccBufs
    const int grp = ew >> 2;
    const int sub = warp & 3;  // TMEM lane quarter this warp may access
    for (int it = grp; ok && it < n_tiles; it += 2) {
      const int buf = it % kAccBufs;
      if (!warp_wait(&acc_full[buf], (it / kAccBufs) & 1, p.err, abort_flag)) break;
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
  CSA_TB(3);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int g_index_smem[4][64];

}  // namespace

size_t index_workspace_bytes(int Nq, int E_max, int /*k*/) {
  const size_t stride = (static_cast<size_t>(E_max) + 3) & ~size_t(3);
  return static_cast<size_t>(Nq) * stride * sizeof(float) + 256;
}

cudaError_t launch_index_score(const IndexArgs& a, cudaStream_t s) {
  const int row_bytes = a.Di / 2;
  const int N = std::max(16, (a.Hi + 15) / 16 * 16);
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
  int splits = std::max(1, std::min(tiles_max, 2 * num_sms() / std::max(1, a.Nq)));
  splits = std::max(splits, (tiles_max + kMaxTilesPerCta - 1) / kMaxTilesPerCta);
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

  const size_t smem = 1024 + kStages * 8192 + 4096 + kMaxTilesPerCta * (512 + 256) + 512 + 256 + 512;
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

}  // namespace csa
