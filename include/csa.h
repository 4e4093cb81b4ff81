/*
 * csa.h -- C ABI of libcsa.so: CSA / HCA compressed attention on NVIDIA B200 (sm_100a).
 *
 * The layer (pages: "DeepSeek-V4: Million-Token Context" explainer, CSA and HCA
 * stages; "Follow the white rabbit: DeepSeek V4's architecture in 3D", CSA / HCA /
 * window / indexer paragraphs; "DeepSeek-V4: Towards Highly Efficient
 * Million-Token Context Intelligence" summary, section 2.3):
 *
 *   csa_compress        every m tokens -> one KV entry by per-channel softmax pooling
 *                       (CSA: m = 4, each entry also pools the previous group of 4;
 *                       HCA: m' = 128, no overlap), then RMSNorm and partial RoPE.
 *   csa_compress_step   the same for decode: the entry a new token completes.
 *   csa_norm_rope       RMSNorm + partial RoPE of query heads (and raw window rows).
 *   csa_quantize_mxfp4  FP4 (E2M1, UE8M0 scale per 32) encoding for the lightning indexer.
 *   csa_index_topk      lightning-indexer scores of every visible entry, then top-k
 *                       (csa_index_topk_grouped: queries of one sequence share the key reads).
 *   csa_sparse_attn     shared-KV MQA over the top-k entries plus the raw-token window.
 *   hca_attn            shared-KV MQA over every visible HCA entry plus the window.
 *   csa_sparse_attn_ex, hca_attn_ex  the same with the query's RMSNorm + RoPE applied in the kernel.
 *   csa_grouped_out_proj  grouped projection of the head outputs to the hidden size.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers unless marked "host".  The caller
 *     owns every buffer; the library allocates nothing on these calls.  It keeps a
 *     4-byte device error word per device and, on every device that loads its
 *     module, the fixed 8 MiB scratch array of csa_index_topk_static (resident
 *     whether or not that call is ever made).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Only argument validation is synchronous.  Results are ready when
 *     the stream reaches the call.
 *   - Return codes only: nothing is printed, nothing aborts.  Invalid shapes
 *     give CSA_ERR_INVALID_ARG, shapes outside the supported set
 *     CSA_ERR_UNSUPPORTED, pointers that are not 16-byte aligned
 *     CSA_ERR_ALIGNMENT, a workspace that is too small CSA_ERR_WORKSPACE, a
 *     failed launch CSA_ERR_CUDA.  Faults detected on the device (an index out of
 *     range, a wait that ran out of time) are recorded in the device error word,
 *     read with csa_get_device_error.
 *   - bf16 is IEEE bfloat16 stored as uint16_t; row-major, innermost index last.
 *   - Positions are absolute token positions.  Entry j of a sequence covers
 *     tokens [m*j, m*j+m-1] and sits at position m*(j+1)-1, so a query at
 *     position t sees entries j < floor((t+1)/m): a group is usable once complete;
 *     the window covers the unfinished one.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_H__
typedef struct CUstream_st* cudaStream_t;
#endif

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,
  CSA_ERR_ALIGNMENT = 2,
  CSA_ERR_UNSUPPORTED = 3,
  CSA_ERR_WORKSPACE = 4,
  CSA_ERR_CUDA = 5,
  CSA_ERR_DEVICE = 6
} csa_status;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

/* device error word values (csa_get_device_error) */
#define CSA_DEVERR_NONE 0
#define CSA_DEVERR_TIMEOUT 1   /* a pipeline wait exceeded its bound; the kernel returned early */
#define CSA_DEVERR_INDEX 2     /* an entry index was outside [0, visible entries) and was skipped */


/* Pooling configuration.  CSA: m = 4, overlap = 1; HCA: m = 128, overlap = 0. */
typedef struct {
  int m;            /* tokens per entry, 1..128 */
  int overlap;      /* 1: entry j also pools group j-1 (slots 0..m-1), own group in slots m..2m-1 */
  int C;            /* channels; multiple of 64, at most 1024 */
  int norm;         /* 1: RMSNorm (unit gain) of entries before RoPE */
  float eps;        /* RMSNorm epsilon */
  int rope_dims;    /* partial RoPE on the last rope_dims channels (even, <= C; 0 = none) */
  float rope_theta; /* RoPE base */
  csa_dtype in_dtype;
} csa_pool_cfg;

/*
 * csa_compress -- softmax-weighted pooling of raw KV into compressed entries.
 * ("DeepSeek-V4: Million-Token Context", CSA stage: every m=4 tokens become one
 * entry through a learned softmax weighting; "Follow the white rabbit", CSA
 * paragraph: each entry also draws on the previous group of four; HCA
 * paragraph: weighted averages of 128 tokens with different weights for
 * different parts of the representation, i.e. per channel.)
 *
 *   a[s,c]   = logits[tok_s, c] + slot_bias[s, c]
 *   e[j,c]   = sum_s softmax_s(a[., c])[s] * kv[tok_s, c]   (slots of group j-1 absent for j = 0)
 *   entries  = RoPE_{m(j+1)-1}(RMSNorm(e[j]))  (norm / RoPE per cfg), stored bf16
 *
 * B sequences of T tokens each (kv, logits: [B, T, C], element type cfg->in_dtype);
 * slot_bias: float32 [(1+overlap)*m, C].
 * entries (bf16 [B, E_max, C], may be NULL): entry j of sequence b for j < floor(T/m);
 *   E_max >= floor(T/m).
 * fp4_out / fp4_scale (may be NULL; both or neither): the pooled entries before
 *   norm and RoPE, MXFP4-encoded as in csa_quantize_mxfp4: [B, E_max, C/2] and
 *   [B, E_max, C/32] bytes (the lightning indexer's key cache).
 * window_kv (bf16 [B, T, C], may be NULL): raw-token rows RoPE_u(RMSNorm(kv[u])) used
 *   by the sliding window ("Follow the white rabbit": the most recent 128 tokens
 *   kept separately).
 * Errors: INVALID_ARG for T < 0, B < 1, m outside 1..128, odd rope_dims;
 * UNSUPPORTED for C not a multiple of 64 or > 1024 (fp4 output needs C % 32 == 0).
 */
CSA_API csa_status csa_compress(const csa_pool_cfg* cfg, int B, int T, const void* kv, const void* logits,
                        const float* slot_bias, void* entries, int E_max, uint8_t* fp4_out,
                        uint8_t* fp4_scale, void* window_kv, cudaStream_t stream);

/*
 * csa_compress_step -- the compressor during decode (a token at a time): for each
 * sequence b whose newest token, at position pos[b], completes a group
 * ((pos[b] + 1) % m == 0), entry j = (pos[b] + 1) / m - 1 exactly as csa_compress
 * writes it for the whole sequence (same pooling, norm, RoPE at position pos[b] and
 * MXFP4 key), computed from the sequence's last S = (1 + overlap) * m raw tokens.
 * ("Follow the white rabbit: DeepSeek V4's architecture in 3D", sliding-window
 * paragraph: a group becomes a compressed entry once it is complete, and the tokens of
 * the unfinished group reach attention through the window; so at decode a new entry
 * appears every m-th token.)
 *
 * pos: device int32 [B].  kv, logits: [B, S, C] (cfg->in_dtype), row s holding token
 * pos[b] - S + 1 + s (rows of tokens before position 0 are ignored: entry 0 pools its
 * own group only).  entries / fp4_out / fp4_scale as in csa_compress.  Nothing is
 * written for a sequence whose group is incomplete; an entry index j >= E_max is
 * skipped and flags CSA_DEVERR_INDEX.  The new token's window row is
 * csa_norm_rope of kv at pos[b].
 * Errors: as csa_compress; INVALID_ARG for B < 0, E_max < 1 or a NULL pos / kv / logits.
 */
CSA_API csa_status csa_compress_step(const csa_pool_cfg* cfg, int B, const int32_t* pos, const void* kv,
                                     const void* logits, const float* slot_bias, void* entries, int E_max,
                                     uint8_t* fp4_out, uint8_t* fp4_scale, cudaStream_t stream);

/*
 * csa_norm_rope -- RMSNorm (unit gain) and partial RoPE of `heads` vectors per row
 * ("DeepSeek-V4: Towards Highly Efficient ...", section 2.3 "Other details": RMSNorm
 * on query heads and KV entries right before core attention; dev.to "How DeepSeek-V4
 * Achieves ...": partial rotary positional embedding).
 * x: [rows, heads, C] (dtype), out: bf16 [rows, heads, C].  Row r sits at position
 * pos[r] (device int32 [rows]); pos == NULL means position r % pos_mod.
 * Pairs (2i, 2i+1) of the last rope_dims channels turn by pos * theta^(-2i/rope_dims).
 */
CSA_API csa_status csa_norm_rope(const void* x, csa_dtype dtype, int64_t rows, int heads, int C,
                         const int32_t* pos, int64_t pos_mod, int norm, float eps, int rope_dims,
                         float rope_theta, void* out, cudaStream_t stream);

/*
 * csa_quantize_mxfp4 -- MXFP4 encoding (dev.to "How DeepSeek-V4 Achieves ...": the
 * lightning indexer runs in FP4), per 32-element block of each row:
 *   E = smallest integer with amax <= 6 * 2^E, clamped to [-127, 127] (amax = 0 -> -127);
 *   code = round-half-even(x / 2^E) onto the E2M1 grid {0,.5,1,1.5,2,3,4,6}, sign = sign of x;
 *   scales[r, b] = E + 127; packed[r, i] holds element 2i (low nibble) and 2i+1 (high nibble).
 * x: [rows, cols] (dtype); cols % 32 == 0; packed [rows, cols/2]; scales [rows, cols/32].
 * Bit-exact: the encoding is a pure function of the input bits.
 */
CSA_API csa_status csa_quantize_mxfp4(const void* x, csa_dtype dtype, int64_t rows, int cols, uint8_t* packed,
                              uint8_t* scales, cudaStream_t stream);

/*
 * csa_index_topk -- lightning indexer and top-k selector ("DeepSeek-V4: Million-Token
 * Context", CSA stage: a small attention head scores every compressed block against
 * the query and the top-k selector keeps the best; "Follow the white rabbit", indexer
 * paragraph: low-precision first pass, top 1,024 at maximum context).
 *
 * For query n (sequence q_seq[n], position q_pos[n]) and every visible entry
 * j < n_vis = min(n_entries[q_seq[n]], floor((q_pos[n]+1)/m)):
 *   d[h]  = <deq(q[n,h,:]), deq(k[q_seq[n], j, :])>            (exact in float32)
 *   S[j]  = float32 chain over h = 0..Hi-1: acc = fmaf(w[n,h], max(d[h], 0), acc), acc0 = 0
 * idx_out[n, :] = the k entries with the largest S (ties -> lowest j), ascending,
 * -1 padded; cnt_out[n] = min(k, n_vis).  score_out (optional, [Nq, E_max]) receives S
 * for j < n_vis.
 *
 * q_fp4 [Nq, Hi, Di/2], q_scale [Nq, Hi, Di/32] (csa_quantize_mxfp4 layout); w float32
 * [Nq, Hi]; q_pos, q_seq int32 [Nq]; k_fp4 [B, E_max, Di/2], k_scale [B, E_max, Di/32];
 * n_entries int32 [B].  Supported: Hi in {4, 8, 16, 32, 64}, Di in {64, 128}, 1 <= k <= 2048.
 * workspace: device scratch of csa_index_topk_workspace(Nq, E_max, k) bytes, 256-byte aligned.
 */
CSA_API csa_status csa_index_topk(int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4,
                          const uint8_t* q_scale, const float* w, const int32_t* q_pos,
                          const int32_t* q_seq, int B, int E_max, const uint8_t* k_fp4,
                          const uint8_t* k_scale, const int32_t* n_entries, int32_t* idx_out,
                          int32_t* cnt_out, float* score_out, void* workspace, size_t ws_bytes,
                          cudaStream_t stream);
CSA_API size_t csa_index_topk_workspace(int Nq, int E_max, int k);

/*
 * csa_index_topk_grouped -- csa_index_topk for multi-query decode: several new tokens of
 * one sequence scored together (multi-token-prediction drafts: "DeepSeek-V4: Towards Highly
 * Efficient Million-Token Context Intelligence", section 2, keeps V3's multi-token
 * prediction).  Query rows come in groups of q_group consecutive
 * rows that name the same sequence; every key tile is read once per group and one
 * N = q_group x 64 block-scaled MMA scores all of the group's heads.  Outputs are bitwise
 * those of csa_index_topk on the same rows.
 * Supported: q_group 1 (exactly csa_index_topk) or 2 with Hi = 64 and Di = 128; Nq may
 * be odd (the last group has one row).  A group row that names another sequence than
 * the group's first row records CSA_DEVERR_INDEX and scores -inf for every entry
 * visible to it.  Same workspace as csa_index_topk.
 */
CSA_API csa_status csa_index_topk_grouped(int q_group, int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4,
                                          const uint8_t* q_scale, const float* w, const int32_t* q_pos,
                                          const int32_t* q_seq, int B, int E_max, const uint8_t* k_fp4,
                                          const uint8_t* k_scale, const int32_t* n_entries, int32_t* idx_out,
                                          int32_t* cnt_out, float* score_out, void* workspace, size_t ws_bytes,
                                          cudaStream_t stream);
/* Kernels csa_index_topk launches for these sizes (pre-encoded queries): 1 when the fused
 * decode kernel runs, 2 otherwise (the scoring kernel, then the top-k kernel), 0 for
 * Nq < 1.  See csa_set_index_fusion. */
CSA_API int csa_index_topk_launches(int Nq, int Hi, int Di, int E_max, int k);

/*
 * csa_set_index_fusion -- process-wide switch (off by default) for the fused decode
 * indexer + top-k ("Follow the white rabbit", indexer paragraph: every compressed entry
 * scored, the top 1,024 kept).  With it on, csa_index_topk runs one kernel when a
 * thread-block cluster of 2, 4 or 8 CTAs per query fits (pre-encoded queries, Hi = 64,
 * Di = 128, E_max up to 4 Ki entries per CTA of the cluster, two CTAs per SM and at least
 * as many CTAs as SMs): each CTA scores its slice of the query's entries into shared
 * memory and the cluster selects the top-k there, so the scores never reach global
 * memory.  The results are bit-for-bit those of the two-kernel path; it is off by default
 * because at the 128K decode shape it measures slower (47-51 us against 43.5 us).
 */
CSA_API csa_status csa_set_index_fusion(int on);

/*
 * csa_index_topk_static -- csa_index_topk for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant of the same computation.
 *
 * Who needs it: code that runs the indexer where allocating is not allowed or not
 * wise -- a plugin or custom operator inside a framework that owns every byte of device
 * memory, a serving loop that must never call cudaMalloc (it can synchronise the whole
 * device), a process whose memory a pool reserved up front.  The caller still provides
 * every input and output; the only scratch, the float32 score rows, lives in a fixed
 * 8 MiB device array inside this library, which every GPU that loads the library holds
 * until the process exits.
 *
 * Arguments, results and support limits are those of csa_index_topk, without the
 * workspace.  Size limit: Nq * round_up(E_max, 4) <= 2^21 scores (e.g. 32 queries of
 * 65536 entries); larger calls return CSA_ERR_WORKSPACE and do nothing.
 * The first call on a device looks up the array's device address with that device
 * current; make that first call before any stream capture.  All calls share the one
 * array: two calls that can run at the same time on the GPU (streams without an order
 * between them) race on it.  No part of it has to start at zero: every score a call
 * reads was written earlier by the same call.  Allocates nothing.
 */
CSA_API csa_status csa_index_topk_static(int Nq, int Hi, int Di, int k, int m, const uint8_t* q_fp4,
                                         const uint8_t* q_scale, const float* w, const int32_t* q_pos,
                                         const int32_t* q_seq, int B, int E_max, const uint8_t* k_fp4,
                                         const uint8_t* k_scale, const int32_t* n_entries, int32_t* idx_out,
                                         int32_t* cnt_out, cudaStream_t stream);

/*
 * csa_index_score / csa_topk_select -- the two halves of csa_index_topk, for callers
 * that keep the score rows: csa_index_score writes S (definition above) into
 * scores[n, j] (float32 [Nq, E_stride], E_stride >= E_max) for j < n_vis of query n and
 * leaves the rest of the row untouched; csa_topk_select reads scores[n, 0:n_vis] and
 * writes idx_out / cnt_out exactly as csa_index_topk does.  Same support limits.
 */
CSA_API csa_status csa_index_score(int Nq, int Hi, int Di, int m, const uint8_t* q_fp4, const uint8_t* q_scale,
                                   const float* w, const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                                   const uint8_t* k_fp4, const uint8_t* k_scale, const int32_t* n_entries,
                                   float* scores, int E_stride, cudaStream_t stream);
/*
 * csa_index_score_q -- csa_index_score taking the indexer queries unencoded:
 * q [Nq, Hi, Di] in q_dtype (CSA_F32 or CSA_BF16), row-major, 8-byte aligned (f32) or
 * 4-byte aligned (bf16).  Each query is encoded to MXFP4 inside the indexer by the rule
 * of csa_quantize_mxfp4 (same bytes), so the scores equal csa_quantize_mxfp4 followed by
 * csa_index_score; the encoded query is not written out.  Same support limits.
 */
CSA_API csa_status csa_index_score_q(int Nq, int Hi, int Di, int m, const void* q, csa_dtype q_dtype, const float* w,
                                     const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                                     const uint8_t* k_fp4, const uint8_t* k_scale, const int32_t* n_entries,
                                     float* scores, int E_stride, cudaStream_t stream);
CSA_API csa_status csa_topk_select(int Nq, int k, int m, const float* scores, int E_stride, const int32_t* q_pos,
                                   const int32_t* q_seq, int B, int E_max, const int32_t* n_entries,
                                   int32_t* idx_out, int32_t* cnt_out, cudaStream_t stream);

/*
 * csa_sparse_attn -- core shared-KV MQA of CSA ("DeepSeek-V4: Towards Highly Efficient
 * ...", section 2.3: shared-KV multi-query attention over the k selected entries;
 * "DeepSeek-V4: Million-Token Context": each query head attends to the picked set
 * plus a sliding window of the very recent tokens).
 *
 * For query n at position t in sequence b, keys K_r (= values) are
 *   entries[b, idx[n, r]] for r < cnt[n], then
 *   window_kv[b, u - window_base[b]] for max(0, t-W+1, window_base[b]) <= u <= min(t, window_base[b]+Tw-1),
 * and for each head h one softmax runs over all of them:
 *   out[n,h] = sum_r softmax_r(scale * <q[n,h], K_r>) K_r,   lse[n,h] = log sum_r exp(scale * <q[n,h], K_r>).
 * q bf16 [Nq, H, D] (already normalised and rotated); entries bf16 [B, E_max, D];
 * idx int32 [Nq, k] (entries < 0 or >= E_max are skipped and flag CSA_DEVERR_INDEX);
 * cnt int32 [Nq]; window_kv bf16 [B, Tw, D]; window_base int32 [B]; out bf16 [Nq, H, D];
 * lse float32 [Nq, H] or NULL.  Supported: H == 64, D == 512, W <= 4096.
 * workspace: csa_sparse_attn_workspace(Nq, H, D, k, W) bytes.
 */
CSA_API csa_status csa_sparse_attn(int Nq, int H, int D, int k, int W, float scale, const void* q,
                           const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                           const void* entries, const int32_t* idx, const int32_t* cnt, int Tw,
                           const void* window_kv, const int32_t* window_base, void* out, float* lse,
                           void* workspace, size_t ws_bytes, cudaStream_t stream);
CSA_API size_t csa_sparse_attn_workspace(int Nq, int H, int D, int k, int W);

/*
 * hca_attn -- HCA dense attention ("DeepSeek-V4: Million-Token Context", HCA stage:
 * every query attends to all compressed entries, plain multi-query attention, plus a
 * small sliding window of uncompressed tokens).  As csa_sparse_attn with the selected
 * set replaced by every visible entry j < min(n_entries[b], floor((t+1)/mprime)).
 * workspace: hca_attn_workspace(Nq, H, D, E_max, W) bytes.
 */
CSA_API csa_status hca_attn(int Nq, int H, int D, int mprime, int W, float scale, const void* q,
                    const int32_t* q_pos, const int32_t* q_seq, int B, int E_max, const void* entries,
                    const int32_t* n_entries, int Tw, const void* window_kv, const int32_t* window_base,
                    void* out, float* lse, void* workspace, size_t ws_bytes, cudaStream_t stream);
CSA_API size_t hca_attn_workspace(int Nq, int H, int D, int E_max, int W);

/*
 * Query preparation inside the attention kernels: csa_sparse_attn_ex and hca_attn_ex
 * take the RAW query q (bf16 [Nq, H, D]) and apply the transform of csa_norm_rope
 * (dtype bf16, pos = q_pos) to every head row: RMSNorm with unit gain when norm != 0,
 * then the partial RoPE on the last rope_dims channels.  The kernel rotates those
 * channels in place and folds each head's norm into its logit scale (a rotation commutes
 * with a scale), so the result equals csa_norm_rope followed by csa_sparse_attn /
 * hca_attn up to rounding, without the extra pass over q in HBM.  Supported: rope_dims
 * even, 0 <= rope_dims <= 64.
 */
typedef struct {
  int norm;         /* 1: RMSNorm (unit gain) of each head row */
  float eps;        /* RMSNorm epsilon */
  int rope_dims;    /* partial RoPE on the last rope_dims channels (0 = none) */
  float rope_theta; /* RoPE base */
} csa_q_prep;

/* As csa_sparse_attn / hca_attn, with q raw and prepared in the kernel as `prep` says
 * (prep NULL: q is used as given, i.e. the plain calls).  Same workspace sizes.
 * Errors: as the plain calls; UNSUPPORTED for rope_dims odd, negative or above 64. */
CSA_API csa_status csa_sparse_attn_ex(const csa_q_prep* prep, int Nq, int H, int D, int k, int W, float scale,
                                      const void* q, const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                                      const void* entries, const int32_t* idx, const int32_t* cnt, int Tw,
                                      const void* window_kv, const int32_t* window_base, void* out, float* lse,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream);
CSA_API csa_status hca_attn_ex(const csa_q_prep* prep, int Nq, int H, int D, int mprime, int W, float scale,
                               const void* q, const int32_t* q_pos, const int32_t* q_seq, int B, int E_max,
                               const void* entries, const int32_t* n_entries, int Tw, const void* window_kv,
                               const int32_t* window_base, void* out, float* lse, void* workspace, size_t ws_bytes,
                               cudaStream_t stream);

/*
 * csa_grouped_out_proj -- grouped output projection of the core-attention outputs back to
 * the hidden size ("DeepSeek-V4: Towards Highly Efficient Million-Token Context
 * Intelligence", section 2.3, "Shared KV and output projection": CSA and HCA project their
 * many head outputs through a grouped projection, cheaper than one dense projection).
 * The H heads form G groups of H/G consecutive heads:
 *   z[t, g R + r] = sum_i o[t, g (H/G) D + i] A[g, r, i]      (i < (H/G) D; group g's own matrix)
 *   y[t, n]       = sum_j z[t, j] Bm[n, j]                    (j < G R)
 * o bf16 [T, H, D] (the attention output layout); A bf16 [G, R, (H/G) D]; Bm bf16
 * [d_model, G R]; z bf16 [T, G R] (the intermediate, written, caller-owned); y bf16
 * [T, d_model].  float32 accumulation; z is rounded to bf16 before the second product.
 * Supported: (H/G) D a multiple of 64, R and d_model multiples of 256.  Two tcgen05 GEMM
 * launches on `stream`.
 */
CSA_API csa_status csa_grouped_out_proj(int T, int H, int D, int G, int R, int d_model, const void* o, const void* A,
                                        const void* Bm, void* z, void* y, cudaStream_t stream);

/* Synchronises `stream`, returns the device error word of the current device in
 * *code_out and clears it.  CSA_ERR_CUDA if the stream reports an error. */
CSA_API csa_status csa_get_device_error(int32_t* code_out, cudaStream_t stream);

/*
 * csa_set_batch_invariant -- process-wide switch (off by default) for batch-invariant
 * results.  With it on, csa_sparse_attn and hca_attn split each query's key list into
 * the fewest power-of-two parts of at most 512 rows (at most 8 parts), a rule that
 * depends on k + W (or E_max + W) only.  A query's output is then bitwise the same
 * whatever batch it is computed in, and the decode calls reproduce the prefill's
 * outputs bit for bit.  Every other call is batch-invariant already: indexer scores
 * are a fixed per-pair chain, top-k is exact, and csa_compress_step writes
 * csa_compress's entries.  The workspace sizes follow the setting: query them after
 * setting it.
 */
CSA_API csa_status csa_set_batch_invariant(int on);

/*
 * csa_selftest_bounded_wait -- exercises the failure-detection path of the pipelines:
 * every wait of a kernel in this library on a pipeline barrier gives up after a bounded
 * number of SM cycles (about 2 s), records CSA_DEVERR_TIMEOUT in the device error word
 * and releases the kernel's other roles through a shared abort flag, so a lost arrival
 * ends the kernel instead of hanging the GPU.  This launches one CTA whose two warps wait
 * on barriers that nothing ever completes (sleeping = 1: the suspend-hinted wait of the
 * many-warp roles; 0: the polling wait); warp 1 starts a quarter of the limit later.
 * out (device int64 [4]): per warp, 1 if its wait succeeded (never, here) else 0, then
 * the SM cycles it waited.  Afterwards csa_get_device_error reports CSA_DEVERR_TIMEOUT;
 * the context stays usable.  The pages have no counterpart: this is a test hook.
 */
CSA_API csa_status csa_selftest_bounded_wait(int sleeping, long long* out, cudaStream_t stream);

/*
 * csa_mma_peak_probe -- dense tensor-core throughput probe (a measurement aid; the pages
 * have no counterpart).  `ctas` CTAs (one per SM) each issue `iters` rounds of four
 * tcgen05 MMAs of M = 128, N (16..256, a multiple of 16) and K = 64 block-scaled FP4
 * elements (mxf4 = 1, kind::mxf4.block_scale) or K = 16 bf16 elements (mxf4 = 0,
 * kind::f16) on operands resident in shared memory, so no memory traffic limits the
 * rate.  *flops_out (host, may be NULL) receives the launch's dense FLOPs (2 M N K per
 * MMA); time the call with events on `stream`.  Operand values are a fixed pattern
 * and the output is discarded.
 */
CSA_API csa_status csa_mma_peak_probe(int mxf4, int N, int iters, int ctas, double* flops_out, cudaStream_t stream);

/* Static description of a status code. */
CSA_API const char* csa_status_string(csa_status status);

/* Name and description of the CUDA error behind the calling thread's most recent
 * CSA_ERR_CUDA status (a static string; "no error" if there was none).  Calls that
 * succeed do not clear it. */
CSA_API const char* csa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
