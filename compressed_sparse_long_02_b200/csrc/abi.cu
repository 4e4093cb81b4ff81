// abi.cu -- the extern "C" entry points of libcsa.so (see include/csa.h): argument
// validation, workspace checks, the per-device error word, kernel dispatch.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "csa.h"
#include "internal.h"

namespace csa {
namespace {

__device__ int32_t g_device_error_word;

constexpr int kMaxDevices = 64;
int32_t* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];
std::mutex g_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2_channels(int C) { return C == 64 || C == 128 || C == 256 || C == 512 || C == 1024; }

thread_local cudaError_t g_last_cuda = cudaSuccess;

}  // namespace

csa_status status_from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return CSA_OK;
  if (e == cudaErrorInvalidValue) return CSA_ERR_INVALID_ARG;
  g_last_cuda = e;
  return CSA_ERR_CUDA;
}

namespace {
csa_status from_cuda(cudaError_t e) { return status_from_cuda(e); }
}  // namespace

int32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_err_ptr[dev];
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (g_sms[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = v > 0 ? v : 148;
  }
  return g_sms[dev];
}

}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_last_cuda_error(void) {
  thread_local char buf[256];
  if (g_last_cuda == cudaSuccess) return "no error";
  snprintf(buf, sizeof buf, "%s: %s", cudaGetErrorName(g_last_cuda), cudaGetErrorString(g_last_cuda));
  return buf;
}

csa_status csa_set_index_fusion(int on) {
  set_index_fusion(on != 0);
  return CSA_OK;
}

csa_status csa_set_batch_invariant(int on) {
  set_batch_invariant(on != 0);
  return CSA_OK;
}

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape";
    case CSA_ERR_WORKSPACE: return "workspace too small";
    case CSA_ERR_CUDA: return "CUDA error";
    case CSA_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

csa_status csa_compress(const csa_pool_cfg* cfg, int B, int T, const void* kv, const void* logits,
                        const float* slot_bias, void* entries, int E_max, uint8_t* fp4_out, uint8_t* fp4_scale,
                        void* window_kv, cudaStream_t stream) {
  if (cfg == nullptr || B < 1 || T < 0 || cfg->m < 1 || cfg->m > 128 || (cfg->overlap != 0 && cfg->overlap != 1))
    return CSA_ERR_INVALID_ARG;
  if (cfg->rope_dims < 0 || (cfg->rope_dims & 1) || cfg->rope_dims > cfg->C) return CSA_ERR_INVALID_ARG;
  if (cfg->in_dtype != CSA_F32 && cfg->in_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (!pow2_channels(cfg->C)) return CSA_ERR_UNSUPPORTED;
  if ((fp4_out == nullptr) != (fp4_scale == nullptr)) return CSA_ERR_INVALID_ARG;
  if (kv == nullptr || logits == nullptr || slot_bias == nullptr) return CSA_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(logits) || !aligned16(slot_bias) || !aligned16(entries) || !aligned16(window_kv) ||
      !aligned16(fp4_out) || !aligned16(fp4_scale))
    return CSA_ERR_ALIGNMENT;
  if ((entries != nullptr || fp4_out != nullptr) && E_max < T / cfg->m) return CSA_ERR_INVALID_ARG;
  if (T == 0) return CSA_OK;
  PoolArgs a{};
  a.kv = kv;
  a.logits = logits;
  a.in_bf16 = cfg->in_dtype == CSA_BF16;
  a.bias = slot_bias;
  a.B = B;
  a.T = T;
  a.C = cfg->C;
  a.m = cfg->m;
  a.overlap = cfg->overlap;
  a.norm = cfg->norm;
  a.eps = cfg->eps;
  a.rope_dims = cfg->rope_dims;
  a.theta = cfg->rope_theta;
  a.entries = static_cast<uint16_t*>(entries);
  a.E_max = E_max;
  a.fp4 = fp4_out;
  a.fp4_scale = fp4_scale;
  a.window = static_cast<uint16_t*>(window_kv);  // written in the same pass as the entries
  return from_cuda(launch_pool(a, stream));
}

csa_status csa_compress_step(const csa_pool_cfg* cfg, int B, const int32_t* pos, const void* kv, const void* logits,
                             const float* slot_bias, void* entries, int E_max, uint8_t* fp4_out, uint8_t* fp4_scale,
                             cudaStream_t stream) {
  if (cfg == nullptr || B < 0 || cfg->m < 1 || cfg->m > 128 || (cfg->overlap != 0 && cfg->overlap != 1))
    return CSA_ERR_INVALID_ARG;
  if (cfg->rope_dims < 0 || (cfg->rope_dims & 1) || cfg->rope_dims > cfg->C) return CSA_ERR_INVALID_ARG;
  if (cfg->in_dtype != CSA_F32 && cfg->in_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (!pow2_channels(cfg->C)) return CSA_ERR_UNSUPPORTED;
  if ((fp4_out == nullptr) != (fp4_scale == nullptr)) return CSA_ERR_INVALID_ARG;
  if (B == 0) return CSA_OK;
  if (pos == nullptr || kv == nullptr || logits == nullptr || slot_bias == nullptr || E_max < 1)
    return CSA_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(logits) || !aligned16(slot_bias) || !aligned16(entries) || !aligned16(fp4_out) ||
      !aligned16(fp4_scale))
    return CSA_ERR_ALIGNMENT;
  PoolArgs a{};
  a.kv = kv;
  a.logits = logits;
  a.in_bf16 = cfg->in_dtype == CSA_BF16;
  a.bias = slot_bias;
  a.B = B;
  a.T = 0;
  a.C = cfg->C;
  a.m = cfg->m;
  a.overlap = cfg->overlap;
  a.norm = cfg->norm;
  a.eps = cfg->eps;
  a.rope_dims = cfg->rope_dims;
  a.theta = cfg->rope_theta;
  a.entries = static_cast<uint16_t*>(entries);
  a.E_max = E_max;
  a.fp4 = fp4_out;
  a.fp4_scale = fp4_scale;
  a.pos = pos;
  a.err = device_error_word();
  if (a.err == nullptr) return CSA_ERR_CUDA;
  return from_cuda(launch_pool(a, stream));
}

csa_status csa_norm_rope(const void* x, csa_dtype dtype, int64_t rows, int heads, int C, const int32_t* pos,
                         int64_t pos_mod, int norm, float eps, int rope_dims, float rope_theta, void* out,
                         cudaStream_t stream) {
  if (rows < 0 || heads < 1 || rope_dims < 0 || (rope_dims & 1) || rope_dims > C) return CSA_ERR_INVALID_ARG;
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (pos == nullptr && pos_mod < 1) return CSA_ERR_INVALID_ARG;
  if (!pow2_channels(C)) return CSA_ERR_UNSUPPORTED;
  if (rows > 0 && (x == nullptr || out == nullptr)) return CSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return CSA_ERR_ALIGNMENT;
  if (rows > 2147483647LL) return CSA_ERR_UNSUPPORTED;
  NormRopeArgs a{};
  a.x = x;
  a.in_bf16 = dtype == CSA_BF16;
  a.rows = rows;
  a.heads = heads;
  a.C = C;
  a.pos = pos;
  a.pos_mod = pos_mod;
  a.norm = norm;
  a.eps = eps;
  a.rope_dims = rope_dims;
  a.theta = rope_theta;
  a.out = static_cast<uint16_t*>(out);
  return from_cuda(launch_norm_rope(a, stream));
}

csa_status csa_quantize_mxfp4(const void* x, csa_dtype dtype, int64_t rows, int cols, uint8_t* packed,
                              uint8_t* scales, cudaStream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return CSA_ERR_INVALID_ARG;
  if (dtype != CSA_F32 && dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || packed == nullptr || scales == nullptr)) return CSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales)) return CSA_ERR_ALIGNMENT;
  return from_cuda(launch_quantize_mxfp4(x, dtype == CSA_BF16, rows, cols, packed, scales, stream));
}

int csa_index_topk_launches(int Nq, int Hi, int Di, int E_max, int k) {
  if (Nq < 1) return 0;
  return index_topk_fusable(Nq, Hi, Di, E_max, k, false, nullptr, nullptr) ? 1 : 2;
}

size_t csa_index_topk_workspace(int Nq, int E_max, int k) {
  if (Nq < 0 || E_max < 0) return 0;
  return index_workspace_bytes(Nq, E_max, k);
}

csa_status csa_index_topk(int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4, const uint8_t* q_scale,
                          const float* w, const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                          const uint8_t* k_fp4, const uint8_t* k_scale, const int32_t* n_entries, int32_t* idx_out,
                          int32_t* cnt_out, float* score_out, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return csa_index_topk_grouped(1, Nq, Hi, Di, k, m, q_fp4, q_scale, w, q_pos, q_seq, B, E_max, k_fp4, k_scale,
                                n_entries, idx_out, cnt_out, score_out, workspace, ws_bytes, stream);
}

csa_status csa_index_topk_grouped(int q_group, int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4,
                                  const uint8_t* q_scale, const float* w, const int32_t* q_pos, const int32_t* q_seq,
                                  int B, int E_max, const uint8_t* k_fp4, const uint8_t* k_scale,
                                  const int32_t* n_entries, int32_t* idx_out, int32_t* cnt_out, float* score_out,
                                  void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (Nq < 0 || k < 1 || m < 1 || B < 1 || E_max < 1) return CSA_ERR_INVALID_ARG;
  if (q_group != 1 && q_group != 2) return CSA_ERR_UNSUPPORTED;
  if (q_group == 2 && (Hi != 64 || Di != 128)) return CSA_ERR_UNSUPPORTED;
  if (Hi < 1 || Hi > 64 || (Di != 64 && Di != 128)) return CSA_ERR_UNSUPPORTED;
  if (E_max % 8 != 0) return CSA_ERR_UNSUPPORTED;
  if (Nq == 0) return CSA_OK;
  if (!q_fp4 || !q_scale || !w || !q_pos || !q_seq || !k_fp4 || !k_scale || !n_entries || !idx_out || !cnt_out ||
      !workspace)
    return CSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp4) || !aligned16(k_fp4) || !aligned16(k_scale) || !aligned16(workspace)) return CSA_ERR_ALIGNMENT;
  if (ws_bytes < index_workspace_bytes(Nq, E_max, k)) return CSA_ERR_WORKSPACE;
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
  a.score_out = score_out;
  a.scores_ws = static_cast<float*>(workspace);
  a.E_stride = (E_max + 3) & ~3;
  a.q_group = q_group;
  return from_cuda(launch_index_topk(a, stream));
}

csa_status csa_index_score(int Nq, int Hi, int Di, int m, const uint8_t* q_fp4, const uint8_t* q_scale,
                           const float* w, const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                           const uint8_t* k_fp4, const uint8_t* k_scale, const int32_t* n_entries, float* scores,
                           int E_stride, cudaStream_t stream) {
  if (Nq < 0 || m < 1 || B < 1 || E_max < 1 || E_stride < E_max) return CSA_ERR_INVALID_ARG;
  if (Hi < 1 || Hi > 64 || (Di != 64 && Di != 128)) return CSA_ERR_UNSUPPORTED;
  if (E_max % 8 != 0) return CSA_ERR_UNSUPPORTED;
  if (Nq == 0) return CSA_OK;
  if (!q_fp4 || !q_scale || !w || !q_pos || !q_seq || !k_fp4 || !k_scale || !n_entries || !scores)
    return CSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp4) || !aligned16(k_fp4) || !aligned16(k_scale)) return CSA_ERR_ALIGNMENT;
  IndexArgs a{};
  a.Nq = Nq;
  a.Hi = Hi;
  a.Di = Di;
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
  a.scores_ws = scores;
  a.E_stride = E_stride;
  return from_cuda(launch_index_score(a, stream));
}

csa_status csa_index_score_q(int Nq, int Hi, int Di, int m, const void* q, csa_dtype q_dtype, const float* w,
                             const int32_t* q_pos, const int32_t* q_seq, int B, int E_max, const uint8_t* k_fp4,
                             const uint8_t* k_scale, const int32_t* n_entries, float* scores, int E_stride,
                             cudaStream_t stream) {
  if (Nq < 0 || m < 1 || B < 1 || E_max < 1 || E_stride < E_max) return CSA_ERR_INVALID_ARG;
  if (q_dtype != CSA_F32 && q_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (Hi < 1 || Hi > 64 || (Di != 64 && Di != 128)) return CSA_ERR_UNSUPPORTED;
  if (E_max % 8 != 0) return CSA_ERR_UNSUPPORTED;
  if (Nq == 0) return CSA_OK;
  if (!q || !w || !q_pos || !q_seq || !k_fp4 || !k_scale || !n_entries || !scores) return CSA_ERR_INVALID_ARG;
  if (!aligned16(k_fp4) || !aligned16(k_scale)) return CSA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(q) & (q_dtype == CSA_F32 ? 7u : 3u)) != 0) return CSA_ERR_ALIGNMENT;
  IndexArgs a{};
  a.Nq = Nq;
  a.Hi = Hi;
  a.Di = Di;
  a.m = m;
  a.B = B;
  a.E_max = E_max;
  a.q_raw = q;
  a.q_raw_bf16 = q_dtype == CSA_BF16 ? 1 : 0;
  a.w = w;
  a.q_pos = q_pos;
  a.q_seq = q_seq;
  a.k_fp4 = k_fp4;
  a.k_scale = k_scale;
  a.n_entries = n_entries;
  a.scores_ws = scores;
  a.E_stride = E_stride;
  return from_cuda(launch_index_score(a, stream));
}

csa_status csa_topk_select(int Nq, int k, int m, const float* scores, int E_stride, const int32_t* q_pos,
                           const int32_t* q_seq, int B, int E_max, const int32_t* n_entries, int32_t* idx_out,
                           int32_t* cnt_out, cudaStream_t stream) {
  if (Nq < 0 || k < 1 || m < 1 || B < 1 || E_max < 1 || E_stride < E_max) return CSA_ERR_INVALID_ARG;
  if (Nq == 0) return CSA_OK;
  if (!scores || !q_pos || !q_seq || !n_entries || !idx_out || !cnt_out) return CSA_ERR_INVALID_ARG;
  IndexArgs a{};
  a.Nq = Nq;
  a.k = k;
  a.m = m;
  a.B = B;
  a.E_max = E_max;
  a.q_pos = q_pos;
  a.q_seq = q_seq;
  a.n_entries = n_entries;
  a.idx_out = idx_out;
  a.cnt_out = cnt_out;
  a.scores_ws = const_cast<float*>(scores);
  a.E_stride = E_stride;
  return from_cuda(launch_topk_select(a, stream));
}

size_t csa_sparse_attn_workspace(int Nq, int H, int D, int k, int W) {
  if (Nq < 0 || k < 0 || W < 0) return 0;
  return attn_workspace_bytes(Nq, H, D, k + W);
}

size_t hca_attn_workspace(int Nq, int H, int D, int E_max, int W) {
  if (Nq < 0 || E_max < 0 || W < 0) return 0;
  return attn_workspace_bytes(Nq, H, D, E_max + W);
}

static csa_status attn_common(AttnArgs& a, int max_keys, cudaStream_t stream) {
  if (a.Nq < 0 || a.B < 1 || a.E_max < 0 || a.W < 0 || a.Tw < 0 || !(a.scale > 0.f)) return CSA_ERR_INVALID_ARG;
  if (a.H != 64 || a.D != 512) return CSA_ERR_UNSUPPORTED;
  if (a.W > 4096) return CSA_ERR_UNSUPPORTED;
  if (a.Nq == 0) return CSA_OK;
  if (!a.q || !a.q_pos || !a.q_seq || !a.entries || !a.out || !a.window_base) return CSA_ERR_INVALID_ARG;
  if (a.W > 0 && a.Tw > 0 && a.window == nullptr) return CSA_ERR_INVALID_ARG;
  if (!aligned16(a.q) || !aligned16(a.entries) || !aligned16(a.window) || !aligned16(a.out) || !aligned16(a.ws))
    return CSA_ERR_ALIGNMENT;
  if (a.ws_bytes < attn_workspace_bytes(a.Nq, a.H, a.D, max_keys)) return CSA_ERR_WORKSPACE;
  if (a.window == nullptr) a.window = a.entries;  // never read when Tw == 0 or W == 0
  return from_cuda(launch_attention(a, max_keys, stream));
}

// The query preparation of the _ex calls (NULL: none).
static csa_status set_q_prep(AttnArgs& a, const csa_q_prep* prep) {
  if (prep == nullptr) return CSA_OK;
  if (prep->rope_dims < 0 || prep->rope_dims > 64 || (prep->rope_dims & 1)) return CSA_ERR_UNSUPPORTED;
  if (prep->norm && !(prep->eps >= 0.f)) return CSA_ERR_INVALID_ARG;
  if (prep->rope_dims > 0 && !(prep->rope_theta > 0.f)) return CSA_ERR_INVALID_ARG;
  a.q_prep = 1;
  a.q_norm = prep->norm ? 1 : 0;
  a.q_eps = prep->eps;
  a.rope_dims = prep->rope_dims;
  a.rope_theta = prep->rope_theta;
  return CSA_OK;
}

csa_status csa_sparse_attn(int Nq, int H, int D, int k, int W, float scale, const void* q, const int32_t* q_pos,
                           const int32_t* q_seq, int B, int E_max, const void* entries, const int32_t* idx,
                           const int32_t* cnt, int Tw, const void* window_kv, const int32_t* window_base, void* out,
                           float* lse, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return csa_sparse_attn_ex(nullptr, Nq, H, D, k, W, scale, q, q_pos, q_seq, B, E_max, entries, idx, cnt, Tw,
                            window_kv, window_base, out, lse, workspace, ws_bytes, stream);
}

csa_status csa_sparse_attn_ex(const csa_q_prep* prep, int Nq, int H, int D, int k, int W, float scale, const void* q,
                              const int32_t* q_pos, const int32_t* q_seq, int B, int E_max, const void* entries,
                              const int32_t* idx, const int32_t* cnt, int Tw, const void* window_kv,
                              const int32_t* window_base, void* out, float* lse, void* workspace, size_t ws_bytes,
                              cudaStream_t stream) {
  if (k < 0) return CSA_ERR_INVALID_ARG;
  if (Nq > 0 && k > 0 && (idx == nullptr || cnt == nullptr)) return CSA_ERR_INVALID_ARG;
  AttnArgs a{};
  a.Nq = Nq;
  a.H = H;
  a.D = D;
  a.k = k;
  a.W = W;
  a.scale = scale;
  a.q = static_cast<const uint16_t*>(q);
  a.q_pos = q_pos;
  a.q_seq = q_seq;
  a.B = B;
  a.E_max = E_max;
  a.entries = static_cast<const uint16_t*>(entries);
  a.idx = idx;
  a.cnt = cnt;
  a.dense = 0;
  a.Tw = Tw;
  a.window = static_cast<const uint16_t*>(window_kv);
  a.window_base = window_base;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  const csa_status ps = set_q_prep(a, prep);
  if (ps != CSA_OK) return ps;
  const int max_keys = k + (W < Tw ? W : Tw);
  return attn_common(a, max_keys, stream);
}

csa_status hca_attn(int Nq, int H, int D, int mprime, int W, float scale, const void* q, const int32_t* q_pos,
                    const int32_t* q_seq, int B, int E_max, const void* entries, const int32_t* n_entries, int Tw,
                    const void* window_kv, const int32_t* window_base, void* out, float* lse, void* workspace,
                    size_t ws_bytes, cudaStream_t stream) {
  return hca_attn_ex(nullptr, Nq, H, D, mprime, W, scale, q, q_pos, q_seq, B, E_max, entries, n_entries, Tw, window_kv,
                     window_base, out, lse, workspace, ws_bytes, stream);
}

csa_status hca_attn_ex(const csa_q_prep* prep, int Nq, int H, int D, int mprime, int W, float scale, const void* q,
                       const int32_t* q_pos, const int32_t* q_seq, int B, int E_max, const void* entries,
                       const int32_t* n_entries, int Tw, const void* window_kv, const int32_t* window_base, void* out,
                       float* lse, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (mprime < 1 || (Nq > 0 && n_entries == nullptr)) return CSA_ERR_INVALID_ARG;
  AttnArgs a{};
  a.Nq = Nq;
  a.H = H;
  a.D = D;
  a.k = 0;
  a.W = W;
  a.scale = scale;
  a.q = static_cast<const uint16_t*>(q);
  a.q_pos = q_pos;
  a.q_seq = q_seq;
  a.B = B;
  a.E_max = E_max;
  a.entries = static_cast<const uint16_t*>(entries);
  a.idx = nullptr;
  a.cnt = nullptr;
  a.n_entries = n_entries;
  a.dense = 1;
  a.mprime = mprime;
  a.Tw = Tw;
  a.window = static_cast<const uint16_t*>(window_kv);
  a.window_base = window_base;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  const csa_status ps = set_q_prep(a, prep);
  if (ps != CSA_OK) return ps;
  const int max_keys = E_max + (W < Tw ? W : Tw);
  return attn_common(a, max_keys, stream);
}

csa_status csa_grouped_out_proj(int T, int H, int D, int G, int R, int d_model, const void* o, const void* A,
                                const void* Bm, void* z, void* y, cudaStream_t stream) {
  if (T < 0 || H < 1 || D < 1 || G < 1 || R < 1 || d_model < 1 || H % G != 0) return CSA_ERR_INVALID_ARG;
  if (((H / G) * static_cast<int64_t>(D)) % 64 != 0 || R % 256 != 0 || d_model % 256 != 0) return CSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(H) * D * 2 > (int64_t(1) << 31) || static_cast<int64_t>(G) * R * 2 > (int64_t(1) << 31))
    return CSA_ERR_UNSUPPORTED;
  if (T == 0) return CSA_OK;
  if (!o || !A || !Bm || !z || !y) return CSA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(A) || !aligned16(Bm) || !aligned16(z) || !aligned16(y)) return CSA_ERR_ALIGNMENT;
  GroupedProjArgs a{};
  a.T = T;
  a.H = H;
  a.D = D;
  a.G = G;
  a.R = R;
  a.d_model = d_model;
  a.o = o;
  a.A = A;
  a.Bm = Bm;
  a.z = static_cast<uint16_t*>(z);
  a.y = static_cast<uint16_t*>(y);
  return from_cuda(launch_grouped_out_proj(a, stream));
}

csa_status csa_get_device_error(int32_t* code_out, cudaStream_t stream) {
  if (code_out == nullptr) return CSA_ERR_INVALID_ARG;
  int32_t* d = device_error_word();
  if (d == nullptr) return CSA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return CSA_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, d, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return CSA_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpy(d, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return CSA_ERR_CUDA;
  *code_out = v;
  return CSA_OK;
}

}  // extern "C"
