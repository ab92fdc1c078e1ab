/*
 * gqa_attn — exact grouped-query attention forward for NVIDIA B200 (sm_100a).
 *
 * C ABI of libgqa_attn.so.  Plain pointers and sizes only.
 *
 * What is computed, for b < B, q-head h < Hq, query position i < Sq:
 *
 *   kvh        = h / (Hq / Hk)                  the kv head shared by q-head h's group
 *   allowed(i) = { j < Sk : !causal  or  j <= i + (Sk - Sq) }
 *   s_j        = scale * sum_c q[b,i,h,c] * k[b,j,kvh,c]
 *   out[b,i,h,:] = sum_{j in allowed(i)} exp(s_j) v[b,j,kvh,:] / sum_{j in allowed(i)} exp(s_j)
 *   lse[b,h,i]   = ln sum_{j in allowed(i)} exp(s_j)
 *
 * Sources for the definition:
 *  - "PyTorch 性能分析深度指南 (第三部分)", section "Attention 的计算挑战":
 *    Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V.
 *  - "优化GQA在Flash-Attention中的批量敏感性", section "分组查询注意力的核心设计"
 *    (and "為什么 GQA 推理吞吐先升后降…4 步速查", section "根因"): Hq must be a multiple
 *    of Hk; with Hq=6, Hk=2, q-heads 0,1,2 read kv-head 0 and 3,4,5 read kv-head 1.
 *  - causal=True and softmax_scale = 1/sqrt(d) in every API example of the pages
 *    ("解锁Stable Diffusion效率瓶颈…", section "动态批量调度"; troubleshooting item
 *    "精度下降").
 *  - Readings where the pages are silent: the causal mask is aligned bottom-right
 *    (identical to top-left when Sq == Sk); lse is the natural log over the scaled
 *    scores; a row with no allowed key (only possible when causal and Sq > Sk) gets
 *    out = 0 and lse = -inf.
 *
 * Scheduling variants (results do not depend on them beyond fp32 rounding order):
 *  - pack_gqa: the Hq/Hk query heads of one kv group are folded into the rows of one
 *    128-row tile, so each K/V tile is read once per group ("优化GQA在Flash-Attention中
 *    的批量敏感性", section "Flash-Attention的PackGQA优化"; "為什么 GQA 推理吞吐先升后降…",
 *    section "根因": packing helps when seqlen_q is small or not near a multiple of the
 *    tile height).
 *  - num_splits: the key axis is split into num_splits contiguous ranges computed as
 *    independent partials and merged by an LSE-weighted combine ("為什么 GQA 推理吞吐
 *    先升后降…", section "修復", table rows for large batch: split the K/V axis, then
 *    combine).
 *
 * Layouts (all row-major, contiguous, device memory owned by the caller):
 *   q   bf16 [B, Sq, Hq, d]        k, v  bf16 [B, Sk, Hk, d]
 *   out fp32 [B, Sq, Hq, d]        lse   fp32 [B, Hq, Sq]
 * d must be 64 or 128.  Every pointer must be 16-byte aligned.
 *
 * Threading and ordering: every call is asynchronous on `stream` (a cudaStream_t, or
 * NULL for the legacy default stream) and never synchronises the host.  Calls may be
 * made from several host threads.
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_NULL = 1,     /* a required pointer is NULL                              */
    GQA_ERR_SHAPE = 2,    /* B, Sq, Sk, Hq or Hk < 1, num_splits or pack_gqa invalid, */
                          /* or a tensor larger than the kernel's 32-bit coordinates  */
    GQA_ERR_HEADS = 3,    /* Hq is not a multiple of Hk                              */
    GQA_ERR_HEADDIM = 4,  /* d not in {64, 128}                                      */
    GQA_ERR_ALIGN = 5,    /* a pointer is not 16-byte aligned                         */
    GQA_ERR_ARCH = 6,     /* the current device is not sm_100 (B200 class)           */
    GQA_ERR_ALLOC = 7,    /* split-KV workspace could not be allocated                */
    GQA_ERR_CUDA = 8,     /* a CUDA runtime/driver call failed (launch, tensor map)   */
    GQA_ERR_TIMEOUT = 9,  /* a bounded in-kernel wait ran out (read back by           */
                          /* gqa_attn_device_status after the stream has synchronised) */
    GQA_ERR_SCRATCH = 10  /* gqa_attn_fwd_noalloc: the split-KV partials do not fit the */
                          /* library's static scratch (GQA_NOALLOC_SCRATCH_BYTES)       */
} gqa_status;

/*
 * Forward pass.  Writes out and lse; reads q, k, v.
 *
 *   scale       multiplier of q.k (1/sqrt(d) in the pages' examples); any finite value.
 *   causal      0 or 1.
 *   pack_gqa    -1 = chosen by gqa_attn_choose, 0 = one q-head per tile, 1 = packed.
 *   num_splits  0 = chosen by gqa_attn_choose, >= 1 = that many key ranges.  Clamped to
 *               the number of 128-key blocks and to 16.  With more than one split the
 *               library allocates stream-ordered scratch of gqa_attn_workspace_bytes(...)
 *               bytes from its own per-device memory pool (cudaMallocFromPoolAsync on
 *               `stream`, freed with cudaFreeAsync after the combine on the same stream;
 *               the pool keeps freed memory for reuse until the process exits).
 *
 * Errors: argument errors return before anything is launched or written.  Launch
 * errors return GQA_ERR_CUDA.  A device-side bounded-wait timeout (which should not
 * happen) is reported through gqa_attn_device_status.
 */
GQA_API gqa_status gqa_attn_fwd(const void* q, const void* k, const void* v, float* out, float* lse,
                        int B, int Sq, int Sk, int Hq, int Hk, int d, float scale, int causal,
                        int pack_gqa, int num_splits, void* stream);

/*
 * The scheduling heuristic alone (no launch, no allocation): what gqa_attn_fwd uses when
 * pack_gqa = -1 / num_splits = 0.  num_sms is the SM count to plan for (148 on B200);
 * num_sms <= 0 plans for the current CUDA device's count, as gqa_attn_fwd does, or for
 * 148 when no device is available (the only CUDA calls made are the device queries).
 * Compared with the pages' call, which takes tensors and decides inside, this entry point
 * also takes Hk, causal and num_sms, because the rule depends on the group size, the mask
 * and the number of SMs to fill.
 *
 * The pages give four mutually contradictory batch-size tables tuned on H100
 * ("解锁Stable Diffusion效率瓶颈…", "动态批量调度" and "三步优化检查清单";
 * "优化GQA在Flash-Attention中的批量敏感性", strategy 2 and "参数组合"; "為什么 GQA 推理吞吐
 * 先升后降…", "修復" table); this rule is re-derived for B200 instead: pack when it
 * computes fewer padded tile rows (causal: also at equal rows, since the two packed tiles
 * of a unit then end on the same key block), split the key axis when the (batch, head,
 * q-tile) units alone cannot fill the SMs.
 *
 * Tuned schedules replace the rule.  The table (written by the package's autotune module;
 * read once per process, at the first call that needs it) is the file named by the
 * environment variable GQA_TUNE_TABLE or, when that variable is unset, tune_b200.txt in the
 * directory of this library: the table shipped with it, measured on B200 over the
 * benchmark workloads.  GQA_TUNE_TABLE set to the empty string turns tuning off.  A shape
 * whose bucket (d, causal, Hq, Hk and the power-of-two buckets of B, Sq, Sk) has an entry
 * gets that entry's pack_gqa / num_splits, validated for the shape (packing needs
 * Hq/Hk <= 128; splits are clamped to the key blocks).  The same applies to gqa_attn_fwd
 * called with pack_gqa = -1 and num_splits = 0; not to gqa_attn_fwd_kvcache with
 * per-sequence lengths.  A missing or unreadable file leaves the rule in place.
 */
GQA_API gqa_status gqa_attn_choose(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal,
                           int num_sms, int* pack_gqa, int* num_splits);

/* Bytes of split-KV scratch gqa_attn_fwd allocates for these arguments (0 when
 * num_splits resolves to 1): num_splits * B * Hq * Sq * (d + 1) * 4 after num_splits is
 * resolved.  pack_gqa / num_splits follow gqa_attn_fwd's conventions; an automatic split
 * count is resolved for the current device's SM count (148 without a device), exactly as
 * gqa_attn_fwd resolves it.  It takes Sk, Hk, causal and pack_gqa besides (B, Sq, Hq, d,
 * num_splits) because an automatic split count depends on all of them.  Invalid arguments
 * give 0. */
GQA_API size_t gqa_attn_workspace_bytes(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal,
                                int pack_gqa, int num_splits);

/* Element type of the output of gqa_attn_fwd_kvcache. */
typedef enum { GQA_OUT_F32 = 0, GQA_OUT_BF16 = 1 } gqa_out_dtype;

/*
 * gqa_attn_fwd_kvcache — the forward of gqa_attn_fwd against a KV cache whose sequences
 * have their own lengths, with an fp32 or bf16 output.
 *
 * The pages run GQA inference against a KV cache that grows with autoregressive
 * generation ("手把手教你理解Llama2的GQA", section "2.1 KV缓存的内存优化"; "PyTorch 性能分析
 * 深度指南 (第三部分)", section "深度剖析：内存瓶颈与 KV Cache"), over sequences of different
 * lengths ("解锁Stable Diffusion效率瓶颈…", section "行业应用场景拓展", scenario one), and
 * recommend BF16 for attention throughput ("PyTorch 性能分析深度指南", closing advice
 * "混合精度").
 *
 *   k_cache, v_cache  bf16 [B, Sk, Hk, d] as k and v of gqa_attn_fwd; Sk is the cache's
 *                     capacity per sequence.
 *   cache_seqlens     device int32 [B] or NULL.  Sequence b uses keys [0, L_b) with
 *                     L_b = cache_seqlens[b] clamped to [0, Sk]; rows past L_b are never
 *                     read into the result.  NULL: L_b = Sk for every b (then this call
 *                     equals gqa_attn_fwd with the chosen output type).  Read by the
 *                     kernels on the device, in stream order; must stay valid until the
 *                     call's work on the stream is done.
 *   causal            bottom-right aligned to each sequence's own length: query i of
 *                     sequence b sees key j iff j < L_b and j <= i + L_b - Sq.  A row with
 *                     no key (e.g. L_b = 0) gets O = 0 and LSE = -inf.
 *   out               [B, Sq, Hq, d], fp32 (out_dtype GQA_OUT_F32) or bf16 rounded to
 *                     nearest even (GQA_OUT_BF16); 16-byte aligned.
 *   out_dtype         GQA_OUT_F32 or GQA_OUT_BF16; anything else returns GQA_ERR_SHAPE.
 *   lse               fp32 [B, Hq, Sq] as in gqa_attn_fwd.
 *   other arguments   as gqa_attn_fwd.  The heuristic sizes splits for the capacity Sk.
 *
 * Errors as gqa_attn_fwd, plus GQA_ERR_ALIGN for a cache_seqlens pointer that is not
 * 4-byte aligned.  Split-KV partials stay fp32 (allocated as for gqa_attn_fwd).  With
 * cache_seqlens given and num_splits = 0, the split count follows a rule for ragged
 * lengths (about three work units per CTA slot), so the partials can differ from what
 * gqa_attn_workspace_bytes reports for the same shape; at most 16 splits of
 * B * Hq * Sq * (d + 1) fp32 values.  With cache_seqlens given and a short query axis
 * (one 128-row tile of rows per (sequence, head or group): decode), a small pre-pass on
 * the device orders the work units by their key count, longest first, and deals them over
 * the CTAs; its scratch is 8 bytes per work unit, taken with the partials from the same
 * pool.  The order changes which CTA computes a unit, never the result.
 */
GQA_API gqa_status gqa_attn_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache,
                                        const int* cache_seqlens, void* out, int out_dtype,
                                        float* lse, int B, int Sq, int Sk, int Hq, int Hk, int d,
                                        float scale, int causal, int pack_gqa, int num_splits,
                                        void* stream);

/*
 * gqa_attn_fwd_paged — the forward of gqa_attn_fwd_kvcache against a paged KV cache: the
 * keys and values of every sequence live in fixed-size pages of a shared pool, found
 * through a block table, instead of one dense [B, Sk, Hk, d] slab.
 *
 * The pages name a paged KV cache for sequences of changing length ("解锁Stable Diffusion
 * 效率瓶颈…", section "行业应用场景拓展", scenario one: 分页KV缓存) and as the remedy when
 * memory runs out for sequences longer than 8192 ("解锁Stable Diffusion效率瓶颈…", section
 * "常见问题排查流程图", item 2 "内存溢出").
 *
 *   k_pages, v_pages   bf16 [num_pages, page_size, Hk, d], row-major, 16-byte aligned: the
 *                      page pools.
 *   block_table        device int32 [B, max_pages_per_seq], 4-byte aligned.  Key j of
 *                      sequence b is row j % page_size of page
 *                      block_table[b * max_pages_per_seq + j / page_size].  Only the entries
 *                      of pages that hold a key j < L_b are used; an entry outside
 *                      [0, num_pages) reads as a page of zeros (no fault).
 *   cache_seqlens      device int32 [B], required.  Sequence b has L_b keys, L_b =
 *                      cache_seqlens[b] clamped to [0, max_pages_per_seq * page_size].
 *   page_size          a power of two >= 16 (e.g. 16, 64, 256).
 *   other arguments    as gqa_attn_fwd_kvcache, with Sk = max_pages_per_seq * page_size.
 *
 * The keys of a page past L_b but in the page that holds key L_b - 1 are read by the
 * kernel (masked out of the result); like the dense cache's rows past L_b, they must hold
 * finite values.  Read on the device in stream order; the table and lengths must stay
 * valid until the call's work on the stream is done.
 *
 * Errors as gqa_attn_fwd_kvcache; GQA_ERR_NULL for a NULL block_table or cache_seqlens;
 * GQA_ERR_SHAPE for a page_size that is not a power of two >= 16, num_pages or
 * max_pages_per_seq < 1, or a pool with 2^31 rows or more; GQA_ERR_ALIGN for a
 * misaligned block_table.
 */
GQA_API gqa_status gqa_attn_fwd_paged(const void* q, const void* k_pages, const void* v_pages,
                                      const int* block_table, int max_pages_per_seq,
                                      const int* cache_seqlens, int num_pages, int page_size,
                                      void* out, int out_dtype, float* lse, int B, int Sq, int Hq,
                                      int Hk, int d, float scale, int causal, int pack_gqa,
                                      int num_splits, void* stream);

/*
 * gqa_attn_fwd_fp8 — the forward of gqa_attn_fwd_kvcache with 8-bit inputs: Q, K and V
 * in e4m3 (OCP FP8 E4M3: 4 exponent bits, bias 7, 3 mantissa bits, largest finite 448)
 * with one fp32 scale per tensor.
 *
 * The pages recommend FP8 for the intermediate computation to halve the bandwidth
 * pressure of attention ("解锁Stable Diffusion效率瓶颈…", "行业应用场景拓展", scenario two,
 * "FP16输入，FP8中间计算"; "三步优化检查清单", step one; "為什么 GQA 推理吞吐先升后降…",
 * "驗證與進階"; "PyTorch 性能分析深度指南 (第三部分)", "总结与建议", 混合精度).
 *
 *   q, k, v             e4m3 bytes, [B, Sq, Hq, d] and [B, Sk, Hk, d], 16-byte aligned.
 *   q_scale, k_scale, v_scale   finite, > 0: the inputs stand for q * q_scale, k * k_scale
 *                       and v * v_scale, and the result is the attention of those values.
 *   cache_seqlens       NULL, or per-sequence key counts as in gqa_attn_fwd_kvcache.
 *   other arguments     as gqa_attn_fwd_kvcache (fp32 or bf16 out, fp32 lse).
 *
 * How it computes: Q K^T in e4m3 with fp32 accumulation; the softmax in fp32 as for bf16
 * inputs; P rounded to e4m3 (to nearest even) for P V, also with fp32 accumulation.  The
 * row sums keep the unrounded P, and each row's largest p is at least 1/2.  Relative to the
 * exact attention of the scaled inputs, an output element's error is then at most
 * 2^-4 * sum_j w_j |v_j| + 2^-9 * max_j w_j * sum_j |v_j| (w_j the exact softmax weights)
 * plus fp32 rounding; the LSE carries only fp32 rounding.
 *
 * Errors as gqa_attn_fwd_kvcache; GQA_ERR_SHAPE also for a scale that is not finite and
 * positive.
 */
GQA_API gqa_status gqa_attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale,
                                    float k_scale, float v_scale, const int* cache_seqlens,
                                    void* out, int out_dtype, float* lse, int B, int Sq, int Sk,
                                    int Hq, int Hk, int d, float scale, int causal, int pack_gqa,
                                    int num_splits, void* stream);

/* Static description of a status code. */
GQA_API const char* gqa_attn_status_string(gqa_status status);

/*
 * Device-side status word of the current device (GQA_OK or GQA_ERR_TIMEOUT), written by
 * kernels whose bounded waits ran out.  Synchronous: it waits for the device.  With
 * reset != 0 the word is cleared after reading.
 *
 * Every wait inside the forward kernel (for a copy, an MMA or another warp's hand-off) is
 * bounded.  The limit is read at each call from the environment: GQA_WAIT_TIMEOUT_NS
 * (nanoseconds) if set, else GQA_WAIT_TIMEOUT_MS (milliseconds), else 4 s.  A CTA whose
 * wait runs out sets this word, stops issuing work, lets the copies and MMAs it already
 * issued complete (waiting at least 1 s for them, whatever the limit), releases its
 * tensor memory and exits; the rest of the grid notices and exits the same way.  The
 * call itself has already returned GQA_OK (it is asynchronous), and out / lse are then
 * partly unwritten: read this word after synchronising when that matters.  Later calls
 * are unaffected.  With GQA_FAULT_INJECT_STALL set (tests of this path), every CTA first
 * waits on a barrier that nothing completes, so the limit runs out on purpose; the GPU
 * stays healthy and the next call without it runs normally.
 */
GQA_API gqa_status gqa_attn_device_status(int reset);

/*
 * gqa_attn_fwd_noalloc — the same forward as gqa_attn_fwd, with the same arguments and
 * results, for callers that must not allocate device memory.  (The pages have no
 * counterpart; this is an interface addition of this library.)
 *
 * Who needs it: a serving process that reserves nearly all device memory up front
 * (weights, KV-cache pools) and forbids any allocation on its hot path, so an
 * allocation there can fail mid-step with nothing to fall back on; code that must not
 * make a call that may block on the device, as cudaMalloc/cudaFree can; and hosts
 * that embed this library under another runtime's allocator, which owns device memory
 * and does not expect a library to grab some of it behind its back.  gqa_attn_fwd
 * allocates the split-KV partials with cudaMallocAsync when num_splits > 1; this entry
 * point never allocates.
 *
 * Scratch: the split-KV partials (O_s and lse_s per split) live in one fixed array
 * inside the library, GQA_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads the
 * library, held until the process exits.  The partials need
 * num_splits * B * Hq * Sq * (d + 1) * 4 bytes.  With num_splits = 0 (automatic) the
 * chosen split count is lowered until they fit, down to 1, which needs no scratch; so an
 * automatic call never fails for lack of scratch (it may run with fewer splits than
 * gqa_attn_fwd would).  An explicit num_splits whose partials do not fit returns
 * GQA_ERR_SCRATCH before anything is launched.
 *
 * The array is shared by every call on a device and keeps the last call's contents.
 * Nothing in it has to start at zero: every partial element is written before the
 * combine reads it.  Calls whose kernels overlap on the GPU (different streams, or
 * different host threads without ordering between them) race on the array; order them
 * on one stream or with events.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current.  Make that first call before any
 * stream capture on the device.  A failed look-up returns GQA_ERR_CUDA.
 */
#define GQA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

GQA_API gqa_status gqa_attn_fwd_noalloc(const void* q, const void* k, const void* v, float* out,
                                        float* lse, int B, int Sq, int Sk, int Hq, int Hk, int d,
                                        float scale, int causal, int pack_gqa, int num_splits,
                                        void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
