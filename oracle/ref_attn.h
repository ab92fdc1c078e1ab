/*
 * fp64 CPU oracle for exact grouped-query attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this
 * code: only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code with the CUDA path.
 *
 * What it computes (the plain two-pass definition, no blocking, no online softmax):
 *
 *   Attention(Q,K,V) = softmax(scale * Q K^T) V                 [1]
 *   q-head h reads kv-head  h / (Hq/Hk),   Hq % Hk == 0         [2]
 *   causal: key j is allowed for query row i iff j <= i + (Sk - Sq)   (reading R4)
 *   LSE[b,h,i] = ln sum_{j allowed} exp(scale * q_i . k_j)      (reading R3)
 *   a row with no allowed key: O = 0, LSE = -inf                  (reading R5)
 *   split-KV combine of partials (O_s, lse_s) over disjoint key ranges:
 *       M = max_s lse_s;  w_s = exp(lse_s - M);  lse = M + ln sum w_s;
 *       O = sum_s w_s O_s / sum_s w_s                            [3]
 *
 * [1] "PyTorch 性能分析深度指南 (第三部分)", section "Attention 的计算挑战": the
 *     scaled dot-product attention formula softmax(QK^T / sqrt(d_k)) V.  The scale is
 *     an argument; 1/sqrt(d) is the pages' default ("解锁Stable Diffusion效率瓶颈",
 *     troubleshooting item "精度下降": softmax_scale = 1/sqrt(d_head)).
 * [2] "优化GQA在Flash-Attention中的批量敏感性", section "分组查询注意力的核心设计":
 *     with Hq=6, Hk=2, q-heads 0,1,2 attend kv-head 0 and 3,4,5 attend kv-head 1;
 *     Hq must be divisible by Hk.
 * [3] "為什么 GQA 推理吞吐先升后降…4 步速查", section "修復" (num_splits row: split
 *     the K/V axis, then combine).  The pages name the combine only; the formula is
 *     the exact merge of softmax partials over disjoint key sets.
 * R3, R4, R5: readings where the pages are silent (listed with the design notes):
 *     the LSE is the natural log over the scaled scores, fp32 on the GPU, [B,Hq,Sq];
 *     the causal mask is aligned bottom-right; an empty row gives O = 0, LSE = -inf.
 *
 * Layouts: Q [B,Sq,Hq,d], K and V [B,Sk,Hk,d] (BSHD, row-major), O [B,Sq,Hq,d],
 * LSE [B,Hq,Sq].  All fp64; callers widen the bf16 inputs exactly.
 */
#ifndef GQA_ORACLE_REF_ATTN_H
#define GQA_ORACLE_REF_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* One query row against one kv-head's keys, restricted to keys [key_lo, key_hi).
 * q: d values.  k, v: key j's row starts at k + j*kv_row_stride (j absolute, 0 <= j < Sk).
 * i: the query's position (0 <= i < Sq), used only by the causal mask. */
void gqa_oracle_row(const double* q, const double* k, const double* v, long kv_row_stride,
                    int d, int Sq, int Sk, int i, double scale, int causal, int key_lo,
                    int key_hi, double* o, double* lse);

/* Whole forward over keys [key_lo, key_hi) (use 0, Sk for the full op).
 * Parallel over (b, h) with OpenMP; returns the number of threads used. */
int gqa_oracle_fwd_range(const double* q, const double* k, const double* v, int B, int Sq,
                         int Sk, int Hq, int Hk, int d, double scale, int causal, int key_lo,
                         int key_hi, double* o, double* lse);

int gqa_oracle_fwd(const double* q, const double* k, const double* v, int B, int Sq, int Sk,
                   int Hq, int Hk, int d, double scale, int causal, double* o, double* lse);

/* Merge split partials.  o_parts [nsplit][rows][d], lse_parts [nsplit][rows];
 * out [rows][d], lse [rows]. */
void gqa_oracle_combine(int nsplit, long rows, int d, const double* o_parts,
                        const double* lse_parts, double* out, double* lse);

#ifdef __cplusplus
}
#endif

#endif
