// noalloc.cu -- csa_index_topk_static: the lightning indexer + top-k with its score
// scratch held in a fixed device array of this library instead of a caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the indexer:
// a plugin or custom operator inside a host framework that owns all device memory and
// forbids allocation during execution, a serving loop that must never call cudaMalloc
// because it can synchronise the whole device and stall other streams, or a process
// whose memory was reserved up front by a pool.  This entry point needs no scratch from
// them: the scores live in g_static_scores below, a file-scope device array that every
// GPU which loads the library holds until the process exits.
//
// The array's device address is resolved once per device, on that device's first call
// (cudaGetSymbolAddress with the device current); host code never passes the array's
// name itself to a kernel, because in host code that name only stands in for the
// device object.  Nothing here calls cudaMalloc, cudaFree or an allocating library.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "csa.h"
#include "internal.h"

namespace csa {
namespace {

constexpr size_t kStaticScoreFloats = size_t(1) << 21;  // 8 MiB of float32 scores

static __device__ __align__(256) float g_static_scores[kStaticScoreFloats];

constexpr int kMaxDevices = 64;
float* g_static_scores_addr[kMaxDevices];
std::mutex g_static_mu;

// Device address of g_static_scores on the current device (resolved on first use) in
// *out; the CUDA result of the lookup (a failure is reported like a failed launch).
cudaError_t static_scores(float** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_scores_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scores);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_static_scores_addr[dev] = static_cast<float*>(p);
  }
  *out = g_static_scores_addr[dev];
  return cudaSuccess;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace csa

extern "C" csa_status csa_index_topk_static(int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4,
                                            const uint8_t* q_scale, const float* w, const int32_t* q_pos,
                                            const int32_t* q_seq, int B, int E_max, const uint8_t* k_fp4,
                                            const uint8_t* k_scale, const int32_t* n_entries, int32_t* idx_out,
                                            int32_t* cnt_out, cudaStream_t stream) {
  using namespace csa;
  if (Nq < 0 || k < 1 || m < 1 || B < 1 || E_max < 1) return CSA_ERR_INVALID_ARG;
  if (Hi < 1 || Hi > 64 || (Di != 64 && Di != 128)) return CSA_ERR_UNSUPPORTED;
  if (E_max % 8 != 0) return CSA_ERR_UNSUPPORTED;
  const int E_stride = (E_max + 3) & ~3;
  if (static_cast<size_t>(Nq) * static_cast<size_t>(E_stride) > kStaticScoreFloats) return CSA_ERR_WORKSPACE;
  if (Nq == 0) return CSA_OK;
  if (!q_fp4 || !q_scale || !w || !q_pos || !q_seq || !k_fp4 || !k_scale || !n_entries || !idx_out || !cnt_out)
    return CSA_ERR_INVALID_ARG;
  if (!is_aligned16(q_fp4) || !is_aligned16(k_fp4) || !is_aligned16(k_scale)) return CSA_ERR_ALIGNMENT;
  float* scratch = nullptr;
  const cudaError_t se = static_scores(&scratch);
  if (se != cudaSuccess) return status_from_cuda(se == cudaErrorInvalidValue ? cudaErrorInvalidSymbol : se);
  IndexArgs a{};
  a.Nq = Nq;
  a.Hi = Hi;
  a.Di = Di;
  a.k = k;
  a.m = m;
  a.B = B;
  a.E_max = E_max;
  a.q_fp4 = q_fp4;
  a.q_scale = q_scale;
  a.w = w;
  a.q_pos = q_pos;
  a.q_seq = q_seq;
  a.k_fp4 = k_fp4;
  a.k_scale = k_scale;
  a.n_entries = n_entries;
  a.idx_out = idx_out;
  a.cnt_out = cnt_out;
  a.score_out = nullptr;
  a.scores_ws = scratch;
  a.E_stride = E_stride;
  return status_from_cuda(launch_index_topk(a, stream));
}
