// internal.h -- host-side declarations shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

#include "csa.h"

namespace csa {

// device error word of the current device (lazily resolved, cached per device)
int32_t* device_error_word();
// Status of a CUDA result; a failure other than cudaErrorInvalidValue is remembered as
// the calling thread's last CUDA error (csa_last_cuda_error) and gives CSA_ERR_CUDA.
csa_status status_from_cuda(cudaError_t e);
int num_sms();

// Raise `fn`'s dynamic shared-memory limit to `bytes` on the current device (once per
// size; `cache` holds the limit already set, one slot per device).
inline cudaError_t set_dyn_smem(const void* fn, size_t bytes, int* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (cache[dev] >= static_cast<int>(bytes)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) cache[dev] = static_cast<int>(bytes);
  return e;
}

// Launch with programmatic stream serialization allowed (kernels call griddep_enter()
// before touching global memory, so an early start is always safe).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same, with the grid's x dimension grouped into thread-block clusters of `cluster`
// consecutive CTAs (1: no clusters).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, unsigned cluster,
                               cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- compressor / norm / rope
struct NormRopeArgs {
  const void* x;
  int in_bf16;
  int64_t rows;
  int heads;
  int C;
  const int32_t* pos;  // nullable
  int64_t pos_mod;
  int norm;
  float eps;
  int rope_dims;
  float theta;
  uint16_t* out;
};
cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s);

struct PoolArgs {
  const void* kv;
  const void* logits;
  int in_bf16;
  const float* bias;
  int B, T, C, m, overlap;
  int norm;
  float eps;
  int rope_dims;
  float theta;
  uint16_t* entries;  // nullable, [B, E_max, C]
  int E_max;
  uint8_t* fp4;       // nullable, [B, E_max, C/2]
  uint8_t* fp4_scale; // nullable, [B, E_max, C/32]
  uint16_t* window;   // nullable, [B, T, C]: RoPE_u(RMSNorm(kv[u])) of every token (not in streaming mode)
  // Streaming (decode) mode when non-null: device [B], the position of each sequence's
  // newest token; kv / logits are then [B, (1+overlap)*m, C], row s holding token
  // pos - (1+overlap)*m + 1 + s, and only the entry that token completes is written.
  const int32_t* pos;
  int32_t* err;       // device error word (streaming mode: an entry index past E_max)
};
cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- MXFP4
cudaError_t launch_quantize_mxfp4(const void* x, int in_bf16, int64_t rows, int cols, uint8_t* packed,
                                  uint8_t* scales, cudaStream_t s);

// ---------------------------------------------------------------- indexer + top-k
struct IndexArgs {
  int Nq, Hi, Di, k, m, B, E_max;
  const uint8_t* q_fp4;
  const uint8_t* q_scale;
  const void* q_raw;  // non-null: unencoded queries [Nq, Hi, Di], encoded to MXFP4 in the indexer
  int q_raw_bf16;
  const float* w;
  const int32_t* q_pos;
  const int32_t* q_seq;
  const uint8_t* k_fp4;
  const uint8_t* k_scale;
  const int32_t* n_entries;
  int32_t* idx_out;
  int32_t* cnt_out;
  float* score_out;  // nullable
  float* scores_ws;  // [Nq, E_stride]
  int E_stride;
  int q_group;       // 2: rows 2g, 2g+1 share a sequence and every key tile (Hi = 64, Di = 128); else 1
};
size_t index_workspace_bytes(int Nq, int E_max, int k);
cudaError_t launch_index_score(const IndexArgs& a, cudaStream_t s);  // writes scores_ws (+ score_out)
cudaError_t launch_topk_select(const IndexArgs& a, cudaStream_t s);  // reads scores_ws
// The fused decode kernel (scores kept on chip, a cluster top-k per query) when the shape
// suits it; *launched tells whether it ran (otherwise nothing was launched).
cudaError_t launch_index_topk_fused(const IndexArgs& a, cudaStream_t s, bool* launched);
bool index_topk_fusable(int Nq, int Hi, int Di, int E_max, int k, bool raw_q, int* C, int* ept);
// The fused decode kernel (process-wide, off by default: measured slower than the two
// kernels at the 128K decode shape).
void set_index_fusion(bool on);
inline cudaError_t launch_index_topk(const IndexArgs& a, cudaStream_t s) {
  bool fused = false;
  cudaError_t e = launch_index_topk_fused(a, s, &fused);
  if (e != cudaSuccess || fused) return e;
  e = launch_index_score(a, s);
  return e != cudaSuccess ? e : launch_topk_select(a, s);
}

// ---------------------------------------------------------------- attention
struct AttnArgs {
  int Nq, H, D, k, W;
  float scale;
  const uint16_t* q;
  const int32_t* q_pos;
  const int32_t* q_seq;
  int B, E_max;
  const uint16_t* entries;
  const int32_t* idx;       // sparse mode; nullptr in dense (HCA) mode
  const int32_t* cnt;       // sparse mode
  const int32_t* n_entries; // dense mode
  int dense;                // 1: every visible entry (HCA); 0: the idx/cnt selection
  int mprime;               // dense mode
  int Tw;
  const uint16_t* window;
  const int32_t* window_base;
  uint16_t* out;
  float* lse;
  void* ws;
  size_t ws_bytes;
  int q_prep;               // 1: q is raw; the kernel applies RMSNorm (q_norm) + partial RoPE
  int q_norm, rope_dims;
  float q_eps, rope_theta;
};
size_t attn_workspace_bytes(int Nq, int H, int D, int max_keys);
// Batch-invariant attention (process-wide, off by default): a query's key list is split
// by a rule that depends on the key count only, never on the batch.
void set_batch_invariant(bool on);
bool batch_invariant();
cudaError_t launch_attention(const AttnArgs& a, int max_keys, cudaStream_t s);

// ---------------------------------------------------------------- grouped output projection
struct GroupedProjArgs {
  int T, H, D, G, R, d_model;
  const void* o;   // bf16 [T, H * D]
  const void* A;   // bf16 [G, R, (H / G) * D]
  const void* Bm;  // bf16 [d_model, G * R]
  uint16_t* z;     // bf16 [T, G * R]
  uint16_t* y;     // bf16 [T, d_model]
};
cudaError_t launch_grouped_out_proj(const GroupedProjArgs& a, cudaStream_t s);

}  // namespace csa
