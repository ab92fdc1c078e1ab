// Parameters shared by the host plan (api.cpp) and the sm_100a kernels.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "fast_divmod.h"

namespace gqa {

constexpr int kBlockM = 128;  // rows of one tile (the tcgen05 M)
constexpr int kBlockN = 128;  // keys of one K/V block
constexpr int kMaxSplits = 16;

// Work unit: one CTA-iteration of the persistent kernel covers NT consecutive tiles of
// one (batch, head-or-group) pair, over one split of the key axis.
struct FwdParams {
    CUtensorMap tm_q;  // q as 4-D (d, Hq, Sq, B); box (64, g or 1, positions, 1)
    CUtensorMap tm_k;  // k as 4-D (d, Hk, Sk, B); box (64, 1, 128, 1)
    CUtensorMap tm_v;  // v likewise
    CUtensorMap tm_o;  // fp32 output for TMA stores: out as (d, Hq, Sq, B), or the split
                       // partials as (d, Hq, Sq, splits*B); box (32, g or 1, positions, 1)

    float* out;       // [B, Sq, Hq, d]       (num_splits == 1)
    float* lse;       // [B, Hq, Sq]          (num_splits == 1)
    float* o_part;    // [splits, B, Sq, Hq, d] (num_splits > 1)
    float* lse_part;  // [splits, B, Hq, Sq]    (num_splits > 1)

    int B, Sq, Sk, Hq, Hk;
    int g;             // Hq / Hk
    int pack;          // 1: a tile holds g heads x pos_per_tile positions
    int pos_per_tile;  // positions one tile covers (packed: floor(128/g); else 128)
    int rows_valid;    // rows of a tile that map to (position, head) (packed: g*pos_per_tile)
    int causal;
    int num_splits;
    int n_hg;          // heads-or-groups per batch: Hq (unpacked) or Hk (packed)
    int n_mt;          // CTA-units along the query axis per (b, hg)
    int n_units;       // n_mt * B * n_hg * num_splits
    int batch_window;  // batches per scheduling window (their K/V fits in L2)
    int kv_blocks;     // ceil(Sk / 128)
    float scale_log2;  // scale * log2(e)
    FastDiv div_g;     // row -> (position, head-in-group) for packed tiles
    // unit index decomposition (see unit_geom): window size, splits, heads-or-groups,
    // batches per full window and in the last (possibly partial) window
    FastDiv div_window, div_splits, div_hg, div_bw, div_bw_last;
    unsigned int* status;  // status word for bounded-wait timeouts (NULL: the library's own)
    long long timeout_ns;  // limit of each in-kernel wait
    long long drain_ns;    // limit of each teardown wait after an abort (>= 1 s)
    // KV cache with per-sequence lengths: keys [0, seqlens_k[b]) of batch b are valid
    // (clamped to [0, Sk]); NULL: every sequence has Sk keys
    const int* seqlens_k;
    // bf16 output [B, Sq, Hq, d] instead of out (num_splits == 1; with splits the combine
    // writes it); NULL: fp32 out.  tm_o then maps it as bf16 with 64-column boxes.
    uint16_t* out_bf16;
    // Paged KV cache (NULL block_table: dense k/v).  tm_k / tm_v then map the page pools
    // [num_pages, page_size, Hk, d] as (d, Hk, page_size, num_pages) with boxes of
    // page_rows = min(page_size, 128) rows; key j of sequence b lies in page
    // block_table[b * table_stride + j / page_size], row j % page_size.
    const int* block_table;
    int table_stride;  // entries per sequence (pages per sequence at most)
    int page_shift;    // log2(page_size)
    int page_rows;     // rows of one TMA box: min(page_size, 128)
    int num_pages;     // pages in the pool (a page coordinate past it reads zeros)
    // Work order (NULL: position u is unit u).  With per-sequence lengths the units' work
    // varies; a pre-pass on the device writes here, for every position u of the static
    // stride, the unit to take there: heaviest first, dealt round by round over the CTAs.
    const int* unit_order;
    // e4m3 inputs: V's per-tensor scale, applied to O in the epilogue (1 for bf16 inputs;
    // Q's and K's scales are folded into scale_log2)
    float v_scale;
    // K/V blocks are read by more than one unit (several query tiles, or unpacked heads,
    // per kv-head): their loads then ask L2 to keep them (evict_last); else they stream
    // (evict_first), like the Q tiles always do
    int kv_shared;
    // fault injection for the failure-detection tests: the producer first waits on a barrier
    // that nothing arrives on, so that the wait limit runs out (GQA_FAULT_INJECT_STALL)
    int inject_stall;
};

struct CombineParams {
    const float* o_part;
    const float* lse_part;
    float* out;
    uint16_t* out_bf16;  // non-NULL: write the output as bf16 here instead of out
    float* lse;
    int B, Sq, Hq, num_splits;
};

}  // namespace gqa
