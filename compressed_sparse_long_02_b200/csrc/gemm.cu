// gemm.cu -- grouped output projection after core attention: the head outputs of each
// group of heads projected by the group's own matrix, then the groups' results
// projected by one dense matrix to the hidden size.
//
// Source: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
// section 2.3, "Shared KV and output projection" (CSA and HCA use a grouped output
// projection, which lowers the cost of bringing many head outputs back to the hidden
// state).  The pages give no sizes; the grouping read here: H heads in G groups of H/G
// consecutive heads, group g's H/G * D outputs times its own [R x (H/G) D] matrix, then
// the G * R results times a [d_model x G R] matrix.
//
// Both stages run one bf16 tcgen05 GEMM kernel, C[:, g Ng + n] = sum_k A[:, g Kg + k] W[g Ng + n, k]
// (row-major A with the group's K slice at column g Kg, stacked per-group weights W, K-major),
// fp32 accumulation in TMEM, bf16 out:
//   stage 1: A = o [T, H D], W = the group matrices [G R, (H/G) D], C = z [T, G R]
//   stage 2: A = z [T, G R], W = the dense matrix [d_model, G R] (one group), C = y [T, d_model]
//
// Persistent CTAs (one per SM) take output tiles of 128 x 256 in turn.  Roles (192
// threads): warp 0 issues TMA loads of the A (128 x 64) and W (256 x 64) slices into a
// 4-stage ring (SWIZZLE_128B, K-major); warp 1 owns TMEM and one thread issues four
// M = 128, N = 256, K = 16 MMAs per stage into one of two 256-column accumulators; warps
// 2-5 drain the other accumulator meanwhile (one TMEM lane quarter each: a row of the
// tile per thread, bf16 pack, 16-byte stores).  Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace csa {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;  // bf16 K slice = one 128-byte swizzle row
constexpr int kGStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint32_t kStageA = kBM * kBK * 2;    // 16 KB
constexpr uint32_t kStageB = kBN * kBK * 2;    // 32 KB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr size_t kGemmSmem = 1024 + kGStages * kStageBytes + 256;
static_assert(kGemmSmem <= 227 * 1024, "shared memory budget");

struct GemmParams {
  int M, Kg, Ng, G, ldc;
  int m_blocks, n_blocks, tiles;
  uint16_t* C;
  int32_t* err;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kStageBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* acc_full = empty + kGStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* fin = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_enter();

  const int k_steps = p.Kg / kBK;
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int j = 0;  // stage sequence number
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int per_group = p.m_blocks * p.n_blocks;
        const int g = t / per_group, rem = t % per_group;
        const int m0 = (rem / p.n_blocks) * kBM, n0 = (rem % p.n_blocks) * kBN;
        for (int kb = 0; kb < k_steps; ++kb, ++j) {
          const int s = j % kGStages;
          if (!mbar_wait(&empty[s], ((j / kGStages) & 1) ^ 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + s * kStageBytes);
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(dst, &tm_a, &full[s], (g * p.Kg + kb * kBK) * 2, m0);
          tma_load_2d(dst + kStageA, &tm_w, &full[s], kb * kBK * 2, g * p.Ng + n0);
        }
      }
      // nothing of this CTA's may still be landing when it exits: the last loads issued
      // (already consumed on the normal path) must have completed
      volatile int never = 0;
      for (int i = std::max(0, j - kGStages); i < j; ++i) mbar_wait(&full[i % kGStages], (i / kGStages) & 1, p.err, &never);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
      int j = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++it) {
        const int buf = it & 1;
        if (!mbar_wait(&acc_empty[buf], ((it >> 1) & 1) ^ 1, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + 256 * buf;
        for (int kb = 0; kb < k_steps; ++kb, ++j) {
          const int s = j % kGStages;
          if (!mbar_wait(&full[s], (j / kGStages) & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStageBytes), b0 = a0 + kStageA;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(acc, smem_desc(a0 + 32 * kk, 16, 1024, kSwizzle128B), smem_desc(b0 + 32 * kk, 16, 1024, kSwizzle128B),
                     idesc, (kb | kk) ? 1u : 0u);
          tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(fin);  // every MMA of this thread has completed
      volatile int never = 0;
      mbar_wait(fin, 0, p.err, &never);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5)
    const int quarter = warp & 3;  // the TMEM lanes this warp may read
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      if (!warp_wait_sleep(&acc_full[buf], (it >> 1) & 1, p.err, abort_flag)) break;
      tc_fence_after();
      const int per_group = p.m_blocks * p.n_blocks;
      const int g = t / per_group, rem = t % per_group;
      const int row = (rem / p.n_blocks) * kBM + 32 * quarter + lane;
      const int col0 = g * p.Ng + (rem % p.n_blocks) * kBN;
      uint16_t* crow = p.C + static_cast<size_t>(row) * p.ldc + col0;
#pragma unroll 1
      for (int c = 0; c < kBN; c += 32) {
        uint32_t v[32];
        const uint32_t ta = tmem + lane_base + 256 * buf + c;
        tmem_ld16(ta, v);
        tmem_ld16(ta + 16, v + 16);
        tmem_wait_ld();
        if (row < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(crow + c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the MMA may reuse this accumulator
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int g_gemm_smem[64];

// One launch: C[:, g Ng + n] = A[:, g Kg : (g+1) Kg] . W[g Ng + n, :]^T for g < G.
// A: bf16 [M, G Kg] row-major; W: bf16 [G Ng, Kg]; C: bf16 [M, ldc].
cudaError_t launch_gemm(const void* A, const void* W, uint16_t* C, int M, int Kg, int Ng, int G, int ldc,
                        cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  CUtensorMap tm_a, tm_w;
  if (!encode_2d_u8(&tm_a, A, static_cast<uint64_t>(G) * Kg * 2, static_cast<uint64_t>(M), kBK * 2, kBM,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tm_w, W, static_cast<uint64_t>(Kg) * 2, static_cast<uint64_t>(G) * Ng, kBK * 2, kBN,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.Kg = Kg;
  p.Ng = Ng;
  p.G = G;
  p.ldc = ldc;
  p.m_blocks = (M + kBM - 1) / kBM;
  p.n_blocks = Ng / kBN;
  p.tiles = p.m_blocks * p.n_blocks * G;
  p.C = C;
  p.err = device_error_word();
  if (p.err == nullptr) return cudaErrorUnknown;
  const cudaError_t e = set_dyn_smem(reinterpret_cast<const void*>(gemm_bf16_kernel), kGemmSmem, g_gemm_smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.tiles, num_sms());
  return launch_pdl(gemm_bf16_kernel, dim3(grid), dim3(kGemmThreads), kGemmSmem, s, tm_a, tm_w, p);
}

}  // namespace

cudaError_t launch_grouped_out_proj(const GroupedProjArgs& a, cudaStream_t s) {
  const int Kg = (a.H / a.G) * a.D;
  cudaError_t e = launch_gemm(a.o, a.A, a.z, a.T, Kg, a.R, a.G, a.G * a.R, s);
  if (e != cudaSuccess) return e;
  return launch_gemm(a.z, a.Bm, a.y, a.T, a.G * a.R, a.d_model, 1, a.d_model, s);
}

}  // namespace csa
