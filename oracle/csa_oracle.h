/*
 * csa_oracle.h -- CPU oracle of the CSA / HCA compressed attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow statement of what the
 * layer computes, used to check the CUDA library.  Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may call it; the product path
 * (the CUDA library and its Python binding) never links, imports or runs it.
 *
 * Sources (web pages on DeepSeek-V4; no code exists on them):
 *   [EXPL]  "DeepSeek-V4: Million-Token Context" (codexsims explainer), CSA and HCA stages.
 *   [DEVTO] "How DeepSeek-V4 Achieves Million-Token Contexts Without Quadratic
 *           Attention Costs", section "Two Compression Strategies: CSA and HCA".
 *   [SUMM]  "DeepSeek-V4: Towards Highly Efficient Million-Token Context
 *           Intelligence" (paperlayer summary), section 2.3 "Hybrid Attention
 *           with CSA and HCA" and section 4 "Model Configurations".
 *   [RABBIT] "Follow the white rabbit: DeepSeek V4's architecture in 3D",
 *           paragraphs on HCA, CSA, the sliding window and the lightning indexer.
 *
 * Precision: every floating-point step is double precision, except the
 * indexer's ranking score, which is defined in float32 (see orc_index_scores).
 */
#ifndef CSA_ORACLE_H
#define CSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types of oracle inputs */
enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

/* Number of entries visible to a query at absolute position t.  Entry j covers
 * tokens [m*j, m*j+m-1] and becomes usable once that group is complete, i.e.
 * at position m*(j+1)-1 ([RABBIT]: tokens of an unfinished group are reached
 * only through the window).  Result: min(n_entries, floor((t+1)/m)). */
int64_t orc_n_visible(int64_t t, int m, int64_t n_entries);

/* Softmax-weighted pooling ([EXPL] CSA stage: m=4 tokens -> one entry by a
 * learned softmax weighting; [RABBIT] CSA: each entry also draws on the previous
 * group of four; [RABBIT] HCA: weights differ across parts of the representation,
 * i.e. per channel).
 *   slots(j) = previous group (m tokens, only if overlap and j>0) + own group.
 *   a[s,c]   = z[tok_s, c] + bias[s, c]   (bias row s: 0..m-1 previous group, m..2m-1 own group
 *                                          when overlap; 0..m-1 own group otherwise)
 *   alpha    = softmax over the existing slots, per channel
 *   out[j,c] = sum_s alpha[s,c] * kv[tok_s, c]
 * kv, z: [T, C] of element type in_dt; bias: [(1+overlap)*m, C] float32;
 * out: [floor(T/m), C] double.  Returns the number of entries. */
int orc_pool(int T, int C, int m, int overlap, int in_dt, const void* kv, const void* z,
             const float* bias, double* out);

/* RMSNorm with unit gain ([SUMM] 2.3 "Other details"): x / sqrt(mean(x^2) + eps), in place. */
void orc_rmsnorm(int64_t rows, int C, double eps, double* x);

/* Partial RoPE ([DEVTO]: "Partial Rotary Positional Embedding") on the last
 * rope_dims channels of each row: pair (2i, 2i+1) of that slice is rotated by
 * pos[row] * theta^(-2i/rope_dims).  In place. */
void orc_rope(int64_t rows, int C, int rope_dims, double theta, const int64_t* pos, double* x);

/* MXFP4 encoding of float32 data, 32-element blocks along each row
 * (E2M1 codes, one UE8M0 scale byte per block):
 *   E    = smallest integer with amax <= 6 * 2^E, clamped to [-127, 127]; amax == 0 -> -127
 *   code = round-to-nearest-even of x / 2^E onto {0, 0.5, 1, 1.5, 2, 3, 4, 6}, sign bit = sign of x
 *   scale byte = E + 127; element 2i in the low nibble of byte i.
 * cols must be a multiple of 32.  packed: [rows, cols/2]; scales: [rows, cols/32]. */
void orc_mxfp4_quantize(int64_t rows, int cols, const float* x, uint8_t* packed, uint8_t* scales);

/* Inverse of the encoding: code value * 2^E. */
void orc_mxfp4_dequantize(int64_t rows, int cols, const uint8_t* packed, const uint8_t* scales,
                          double* out);

/* Lightning-indexer scores ([EXPL]: a small attention head scoring every
 * compressed block against the query; [RABBIT]: low-precision first pass adapted
 * from V3.2's sparse attention; [DEVTO]: runs in FP4):
 *   d[h]   = <deq(q[n,h,:]), deq(k[seq(n), j, :])>           (exact)
 *   s64    = sum_h w[n,h] * max(d[h], 0)                      (double)
 *   s32    = float32 chain over h = 0..Hi-1:  acc = fmaf(w[n,h], max((float)d[h], 0), acc), acc0 = +0
 * s32 is the ranking score: the top-k decision is taken on it.  Entries
 * j >= n_vis[n] are left untouched.
 * q_packed [nq,Hi,Di/2], q_scales [nq,Hi,Di/32], w [nq,Hi];
 * k_packed [B,E_max,Di/2], k_scales [B,E_max,Di/32]; s32/s64 [nq,E_max] (s64 may be NULL).
 * Returns the number of per-head dot products that were not exactly
 * representable in float32 (0 for all workloads used here). */
int64_t orc_index_scores(int nq, int Hi, int Di, const uint8_t* q_packed, const uint8_t* q_scales,
                         const float* w, const int32_t* q_seq, const int32_t* n_vis, int E_max,
                         const uint8_t* k_packed, const uint8_t* k_scales, float* s32, double* s64);

/* Top-k selection ([SUMM] 2.3: each query attends only to k compressed entries
 * chosen by the indexer; [RABBIT]: top 1,024 at maximum context).
 * Candidates are j in [0, n_vis[n]).  If n_vis <= k all are taken; otherwise
 * candidates are ordered by (score descending, index ascending) and the first
 * k kept.  Output indices ascending, padded with -1; cnt[n] = number taken.
 * kth (optional, [nq,2]): the k-th and (k+1)-th ordered scores (NaN if n_vis <= k). */
void orc_topk(int nq, int E_stride, const float* scores, const int32_t* n_vis, int k,
              int32_t* idx, int32_t* cnt, float* kth);

/* Core shared-KV MQA ([SUMM] 2.3: shared-KV multi-query attention; [EXPL]: each
 * head attends to the picked set plus a sliding window of recent tokens;
 * [RABBIT]: window of the most recent 128 tokens).  For query n at position t
 * in sequence b, the key set is
 *   { entries[b, idx[n,r]] : r < cnt[n] }  followed by
 *   { window[b, u - wbase[b]] : max(0, t-W+1, wbase[b]) <= u <= min(t, wbase[b]+Tw-1) }
 * and for every head h one softmax runs over the whole set:
 *   p_r = softmax_r(scale * <q[n,h], K_r>),  out[n,h] = sum_r p_r K_r  (K = V),
 *   lse[n,h] = log sum_r exp(scale * <q[n,h], K_r>).
 * An empty key set gives out = 0 and lse = -inf.
 * q [nq,H,D]; entries [B,E_max,D]; window [B,Tw,D] (element types q_dt, e_dt, w_dt);
 * idx [nq,k]; out [nq,H,D] double; lse [nq,H] double (may be NULL). */
void orc_attention(int nq, int H, int D, double scale, int q_dt, const void* q, const int64_t* q_pos,
                   const int32_t* q_seq, int E_max, int e_dt, const void* entries, int k,
                   const int32_t* idx, const int32_t* cnt, int W, int Tw, int w_dt, const void* window,
                   const int64_t* wbase, double* out, double* lse);

/* Grouped output projection ([SUMM] 2.3, "Shared KV and output projection": after core
 * attention, a grouped projection carries the many head outputs back to the hidden state
 * at less cost than one dense projection).  The pages name the grouping but no sizes or
 * structure; the reading taken: the H heads form G groups of H/G consecutive heads; each
 * group's concatenated outputs (H/G * D values) are projected by the group's own matrix
 * to R values; the G * R values are then projected by one dense matrix to d_model:
 *   z[t, g*R + r] = sum_{i < (H/G)*D} o[t, g*(H/G)*D + i] * A[g, r, i]
 *   y[t, n]       = sum_{j < G*R} z[t, j] * Bm[n, j]
 * o [T, H*D], A [G, R, (H/G)*D], Bm [d_model, G*R] (element type in_dt each);
 * z [T, G*R] and y [T, d_model] double.  y is computed from the double z (no rounding
 * of the intermediate).  H must be a multiple of G. */
void orc_grouped_out_proj(int T, int H, int D, int G, int R, int d_model, int in_dt, const void* o, const void* A,
                          const void* Bm, double* z, double* y);

#ifdef __cplusplus
}
#endif
#endif
