// Exact GQA attention forward for sm_100a: persistent, warp-specialised, TMA + tcgen05.
//
// Persistent CTAs walk a static stride of work units: one CTA per SM for two-tile
// units (NT = 2, prefill), two per SM for one-tile units (NT = 1, decode and short query
// axes).  A unit is NT consecutive 128-row query tiles of one (batch, head) pair (or,
// with PackGQA, of one (batch, kv-group) pair whose g query heads are folded into the
// rows), over one split of the key axis.  Roles:
//   warpgroup 0, warp 0   TMA producer: Q tiles once per unit, then a ring of K/V blocks
//                         (a page pool through the block table in the PAGED kernels).
//   warpgroup 0, warp 1   MMA issuer, a converged warp whose elected lane issues:
//                         S_t = Q_t K^T into TMEM (both operands in shared memory), then
//                         O_t += P_t V with P_t read from TMEM.
//   warpgroups 1..NT      softmax, one per tile; thread = tile row = TMEM lane.  Each
//                         reads its S row from TMEM, masks (causal, key tail), keeps the
//                         reference max and row sum, writes P (bf16 or e4m3) over S in
//                         TMEM and rescales O in TMEM when the reference max moves.
//                         At d = 64 with two bf16 tiles, P has TMEM columns of its own
//                         (S and O use 384 of 512), so the MMA issuer starts the next
//                         block's S as soon as the softmax holds this block's S in
//                         registers, ahead of this block's P.V.
//   warpgroup NT + 1      (NT = 2 only) epilogue: O / l through a shared-memory stage and
//                         TMA tensor stores, and the LSE.  With NT = 1 the softmax
//                         warpgroup writes its rows' output itself.
//
// The computation follows the scaled dot-product attention definition
// ("PyTorch 性能分析深度指南 (第三部分)", section "Attention 的计算挑战") with the GQA head
// sharing of "优化GQA在Flash-Attention中的批量敏感性" (section "分组查询注意力的核心设计"),
// the PackGQA row folding of the same page (section "Flash-Attention的PackGQA优化") and
// the split-KV partials of "為什么 GQA 推理吞吐先升后降…4 步速查" (section "修復").
// The online softmax (running max with deferred rescaling) is the standard exact
// reformulation of the row softmax; it reaches the definition up to fp32 rounding.
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <type_traits>

#include "fwd_params.h"
#include "launch.h"
#include "exp2_poly.cuh"
#include "ptx_sm100.cuh"

// Of each 16 exponential pairs of an unmasked 32-key chunk, how many take the FMA-pipe
// polynomial instead of the MUFU; measured per head dimension on B200 (interleaved timing
// of 2-6 pairs): 2 at d=128, 3 at d=64.  -DGQA_EXP_POLY_PAIRS=n overrides both.
#ifdef GQA_EXP_POLY_PAIRS
#define GQA_POLY_PAIRS_FOR(HD) (GQA_EXP_POLY_PAIRS)
#else
#define GQA_POLY_PAIRS_FOR(HD) ((HD) == 128 ? 2 : 3)
#endif

namespace gqa {

__device__ unsigned int g_device_status = 0;

namespace {

using namespace ptx;

// F8: Q, K, V in e4m3 (one byte per element), MMAs of kind::f8f6f4, P in e4m3.
template <int HD, int NT, bool F8 = false>
struct FwdCfg {
    static constexpr int kRowBytes = F8 ? HD : 2 * HD;   // one row of Q, K or V
    // a tile is kChunks column chunks of 128 rows; a chunk row is at most 128 bytes (the
    // swizzle span): bf16 rows split into 64-column chunks, e4m3 rows (64 or 128 bytes) fit
    static constexpr int kChunks = F8 ? 1 : HD / 64;
    static constexpr int kChunkRowBytes = F8 ? kRowBytes : 128;
    static constexpr int kChunkBytes = 128 * kChunkRowBytes;
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kSlots = (F8 ? 2 : 1) * ((NT == 2) ? (HD == 128 ? 4 : 8) : (HD == 128 ? 2 : 5));
    // shared-memory operand layout: 128-byte swizzle (atoms of 8 rows x 128 bytes), or
    // 64-byte swizzle for 64-byte rows
    static constexpr bool kSw64 = kChunkRowBytes == 64;
    static constexpr uint32_t kAtomBytes = 8 * kChunkRowBytes;
    // MMA K per instruction (16 bf16 or 32 e4m3 = 32 bytes) and steps per 128-key P.V
    static constexpr int kMmaK = F8 ? 32 : 16;
    static constexpr int kPvSteps = kBlockN / kMmaK;
    static constexpr uint32_t kPvStepBytes = kMmaK * kChunkRowBytes;  // keys of one step, one chunk
    // TMEM columns of P per 32-key chunk (2 bf16 or 4 e4m3 per column)
    static constexpr int kPColsPer32 = F8 ? 8 : 16;
    // NT == 2: warpgroups 0 = TMA producer + MMA issuer, 1..2 = softmax (one per tile),
    //          3 = epilogue; one CTA per SM.
    // NT == 1: warpgroup 0 as above, 1 = softmax that also writes its tile's output; two
    //          CTAs per SM, so one CTA's unit changes overlap the other's K/V stream.
    static constexpr bool kEpilogueWG = (NT == 2);
    static constexpr int kWarpgroups = 1 + NT + (kEpilogueWG ? 1 : 0);
    static constexpr int kThreads = kWarpgroups * 128;
    static constexpr int kCtasPerSm = kEpilogueWG ? 1 : 2;
    // registers: at launch (65536 / (threads x CTAs), rounded down to 8), then
    // redistributed with setmaxnreg; the per-thread sum over the warpgroups equals
    // warpgroups x launch regs, so every increase is covered by the decreases (each SM
    // sub-partition holds one warp of each warpgroup)
    static constexpr int kLaunchRegs = ((65536 / (kThreads * kCtasPerSm)) / 8) * 8;
    static constexpr int kRegsLoad = NT == 2 ? 104 : 80;
    static constexpr int kRegsSoftmax = NT == 2 ? 168 : 176;
    static constexpr int kRegsEpilogue =
        kEpilogueWG ? kWarpgroups * kLaunchRegs - kRegsLoad - NT * kRegsSoftmax : 0;
    static_assert(kRegsLoad + NT * kRegsSoftmax + kRegsEpilogue == kWarpgroups * kLaunchRegs,
                  "register split must add up to the launch allocation");
    static_assert(!kEpilogueWG || (kRegsEpilogue >= 64 && kRegsEpilogue % 8 == 0),
                  "epilogue registers");
    // of each 16 exponential pairs of a 32-key chunk, this many take the polynomial (unmasked
    // blocks only); the rest use the special-function unit
    static constexpr int kPolyPairs = GQA_POLY_PAIRS_FOR(HD);
    static constexpr int kTmemCols = (NT * 128 + NT * HD) <= 256 ? 256 : 512;
    // d=64 with two tiles (bf16): S and O take 384 of TMEM's 512 columns, which leaves room
    // for P in columns of its own.  The next block's S is then computed while this block's
    // softmax still runs (it needs only the S values already in registers), instead of
    // after this block's P.V.
    static constexpr bool kSepP = (HD == 64 && NT == 2 && !F8);
    static constexpr int kNumBars = 2 * kSlots + 8 * NT + 2 + (kSepP ? 2 * NT : 0);
    static constexpr int kStatsBytes = kEpilogueWG ? 2 * NT * 2 * 128 * 4 : 0;  // (m, l), 2 buffers
    // epilogue staging for TMA stores: 128 rows x 32 fp32 (128 B, swizzled) per chunk
    static constexpr int kOStageBytes = kEpilogueWG ? 128 * 128 : 0;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + NT * kTileBytes +
                                      kSlots * kTileBytes + kOStageBytes + 8 * kNumBars +
                                      kStatsBytes + 16;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static constexpr uint32_t kIdescQK = F8 ? idesc_e4m3_f32(128, 128, false) : idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t kIdescPV = F8 ? idesc_e4m3_f32(128, HD, true) : idesc_bf16_f32(128, HD, true);
    __device__ static uint64_t sdesc(uint32_t saddr, uint32_t lbo) {
        return kSw64 ? sdesc_sw64(saddr, lbo, kAtomBytes) : sdesc_sw128(saddr, lbo, kAtomBytes);
    }
    __device__ static void mma_s(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
        if constexpr (F8) mma_ss_f8(d, a, b, kIdescQK, acc);
        else mma_ss(d, a, b, kIdescQK, acc);
    }
    __device__ static void mma_pv(uint32_t d, uint32_t a, uint64_t b, uint32_t acc) {
        if constexpr (F8) mma_ts_f8(d, a, b, kIdescPV, acc);
        else mma_ts(d, a, b, kIdescPV, acc);
    }
    __host__ __device__ static constexpr int s_col(int t) { return t * 128; }
    __host__ __device__ static constexpr int o_col(int t) { return NT * 128 + t * HD; }
    __host__ __device__ static constexpr int p_col(int t) {
        return kSepP ? NT * 128 + NT * HD + t * 64 : s_col(t);
    }
    // separate P sits this many columns past the tile's O (the same for every tile)
    static constexpr int kPAfterO = NT * HD;
};

template <uint32_t R>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

// Geometry of one work unit, computed identically by every role.
template <int NT>
struct UnitGeom {
    int b, hg, split, kvh;
    int sk;         // keys of this batch element (its KV-cache length, else Sk)
    int pos0[NT];   // first query position of tile t
    int n[NT];      // key blocks tile t processes in this split
    int kb_lo;      // first key block of the split
    int nblk;       // max over tiles of n[t]
};

// Unit order: batches are taken in windows of p.batch_window (sized on the host so a
// window's K/V fits in L2); inside a window the query tiles go latest first (the
// heaviest under a causal mask), then batch, then head-or-group, then split.  With a
// static stride over the persistent CTAs this spreads heavy and light tiles evenly and
// keeps every K/V block's readers close together in time.
template <int NT>
__device__ __forceinline__ UnitGeom<NT> unit_geom(int u, const FwdParams& p) {
    // all divisions by run-time sizes are multiply-shift (FastDiv), computed on the host
    if (p.unit_order != nullptr) u = __ldg(p.unit_order + u);
    UnitGeom<NT> g;
    uint32_t w, r, q, rem;
    fastdivmod((uint32_t)u, p.div_window, w, r);
    const int b0 = (int)w * p.batch_window;
    const bool last = b0 + p.batch_window > p.B;
    fastdivmod(r, p.div_splits, q, rem);
    g.split = (int)rem;
    fastdivmod(q, p.div_hg, r, rem);
    g.hg = (int)rem;
    fastdivmod(r, last ? p.div_bw_last : p.div_bw, q, rem);
    g.b = b0 + (int)rem;
    const int mt = p.n_mt - 1 - (int)q;
    g.kvh = p.pack ? g.hg : (int)fastdiv((uint32_t)g.hg, p.div_g);
    g.sk = p.seqlens_k ? min(max(__ldg(p.seqlens_k + g.b), 0), p.Sk) : p.Sk;
    int kb_end[NT];
    int kb_union = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        g.pos0[t] = (mt * NT + t) * p.pos_per_tile;
        kb_end[t] = 0;
        if (g.pos0[t] < p.Sq) {
            int last = min(g.pos0[t] + p.pos_per_tile, p.Sq) - 1;
            // causal: bottom-right aligned to this sequence's own key count
            int key_end = g.sk;
            if (p.causal) key_end = max(0, min(g.sk, last + 1 + (g.sk - p.Sq)));
            kb_end[t] = (key_end + kBlockN - 1) / kBlockN;
        }
        kb_union = max(kb_union, kb_end[t]);
    }
    g.kb_lo = (int)(((long long)g.split * kb_union) / p.num_splits);
    const int kb_hi = (int)(((long long)(g.split + 1) * kb_union) / p.num_splits);
    g.nblk = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        g.n[t] = max(0, min(kb_hi, kb_end[t]) - g.kb_lo);
        g.nblk = max(g.nblk, g.n[t]);
    }
    return g;
}

// a[t] for a run-time t without dynamic indexing (keeps the arrays in registers)
template <int NT>
__device__ __forceinline__ int pick(const int (&a)[NT], int t) {
    int v = a[0];
#pragma unroll
    for (int i = 1; i < NT; ++i) v = (t == i) ? a[i] : v;
    return v;
}

// Row r of tile t of a unit -> (query position, q-head); row_ok when it maps to a real
// output row.  PackGQA: r = position_in_tile * g + head_in_group.
struct RowMap {
    int pos, head;
    bool ok;
};
__device__ __forceinline__ RowMap row_map(const FwdParams& p, int pos0, int hg, int row) {
    RowMap m;
    if (p.pack) {
        uint32_t pr, hh;
        fastdivmod((uint32_t)row, p.div_g, pr, hh);
        m.pos = pos0 + (int)pr;
        m.head = hg * p.g + (int)hh;
        m.ok = row < p.rows_valid && m.pos < p.Sq;
    } else {
        m.pos = pos0 + row;
        m.head = hg;
        m.ok = m.pos < p.Sq;
    }
    return m;
}

// Writes one tile row's output: O / l from TMEM (or zeros for a tile with no key in this
// split) and LSE = (m + log2 l) ln 2, to out/lse or to the split partials.  Arrives on
// o_empty once O is in registers, so the next unit's PV may overwrite it.
template <int HD>
__device__ __forceinline__ void write_row(const FwdParams& p, uint32_t o_addr, const RowMap& rm,
                                          int b, int split, bool has, bool idle, float m, float l,
                                          uint32_t o_empty_bar) {
    constexpr float kLn2 = 0.69314718055994530942f;
    const float inv_l = (l > 0.f) ? p.v_scale / l : 0.f;
    const float lse_v = (l > 0.f) ? (m + __log2f(l)) * kLn2 : -INFINITY;
    float* orow = nullptr;
    float* lrow;
    uint16_t* bf16_row = nullptr;  // bf16 output row (final output only)
    if (p.num_splits == 1) {
        if (p.out_bf16)
            bf16_row = p.out_bf16 + (((size_t)b * p.Sq + rm.pos) * p.Hq + rm.head) * HD;
        else
            orow = p.out + (((size_t)b * p.Sq + rm.pos) * p.Hq + rm.head) * HD;
        lrow = p.lse + ((size_t)b * p.Hq + rm.head) * p.Sq + rm.pos;
    } else {
        const size_t sb = (size_t)split * p.B + b;
        orow = p.o_part + ((sb * p.Sq + rm.pos) * p.Hq + rm.head) * HD;
        lrow = p.lse_part + (sb * p.Hq + rm.head) * p.Sq + rm.pos;
    }
#pragma unroll
    for (int ch = 0; ch < HD / 32; ++ch) {
        uint32_t r[32];
        if (has) {
            if (!idle) {
                ptx::tmem_ld32(o_addr + ch * 32, r);
                ptx::tmem_wait_ld();
            }
            if (ch == HD / 32 - 1) {
                ptx::tc_fence_before();
                ptx::mbar_arrive(o_empty_bar);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        if (rm.ok && bf16_row != nullptr) {
            uint4* dst = reinterpret_cast<uint4*>(bf16_row + ch * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(
                    ptx::pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l),
                    ptx::pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l),
                    ptx::pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l),
                    ptx::pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l));
        } else if (rm.ok) {
            float4* dst = reinterpret_cast<float4*>(orow + ch * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(r[4 * i + 0]) * inv_l,
                                     __uint_as_float(r[4 * i + 1]) * inv_l,
                                     __uint_as_float(r[4 * i + 2]) * inv_l,
                                     __uint_as_float(r[4 * i + 3]) * inv_l);
        }
    }
    if (rm.ok) *lrow = lse_v;
}

// Paged KV: the block-table entries of one sequence, cached in the producer warp's
// registers 32 at a time (lane i holds entry base + i), with the next 32 already loaded
// (lane i of w1 holds base + 32 + i) so that moving on does not wait for memory.
// Warp-collective: every lane calls it with the same arguments.
struct PageCache {
    int b = -1;
    int base = 0;
    int w0 = -1, w1 = -1;
};
__device__ __forceinline__ int table_entry(const FwdParams& p, int b, int i) {
    return (i < p.table_stride) ? __ldg(p.block_table + (size_t)b * p.table_stride + i) : -1;
}
__device__ __forceinline__ int page_of(PageCache& pc, const FwdParams& p, int b, int page_i,
                                       int lane) {
    if (b != pc.b || page_i < pc.base || page_i >= pc.base + 64) {
        pc.b = b;
        pc.base = page_i & ~31;
        pc.w0 = table_entry(p, b, pc.base + lane);
        pc.w1 = table_entry(p, b, pc.base + 32 + lane);
    } else if (page_i >= pc.base + 32) {
        pc.base += 32;
        pc.w0 = pc.w1;
        pc.w1 = table_entry(p, b, pc.base + 32 + lane);
    }
    return __shfl_sync(0xffffffffu, pc.w0, page_i - pc.base);
}

// Bounded wait on an mbarrier phase.  Returns false when the CTA is aborting or when
// this wait ran past the time limit (then it records the timeout and starts the abort).
// Suspending probes (try_wait); the clock and the abort flag are read every 256 of them.
// The code inlined at each wait site is kept this small on purpose: a larger inlined wait
// (a second, test-only probe loop) measured 4-7 % slower prefill, the hot loops' code
// sharing the SM's instruction cache with every wait site.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile uint32_t* abort_flag,
                                             const FwdParams& p) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer();
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
        if ((++spins & 255u) == 0) {
            if (*abort_flag) return false;
            if ((long long)(globaltimer() - t0) > p.timeout_ns) {
                *abort_flag = 1u;
                atomicOr(p.status ? p.status : &g_device_status, 1u);
                return false;
            }
        }
    }
    return true;
}

// Wait used during teardown: ignores the abort flag, gives up silently at its own limit
// (p.drain_ns, at least 1 s: copies and MMAs already issued finish in microseconds, and
// they must land before the CTA's shared and tensor memory are released).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, const FwdParams& p) {
    uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if ((long long)(globaltimer() - t0) > p.drain_ns) return;
    }
}

// PAGED: K/V come from page pools through the block table (the producer's address
// computation only; a separate instantiation, so the dense kernels carry none of it in
// their instruction stream).
template <int HD, int NT, bool F8, bool PAGED>
__global__ void __launch_bounds__(FwdCfg<HD, NT, F8>::kThreads, FwdCfg<HD, NT, F8>::kCtasPerSm)
    gqa_fwd_kernel(const __grid_constant__ FwdParams p) {
    using C = FwdCfg<HD, NT, F8>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);

    const uint32_t sQ = base;
    const uint32_t sKV = base + NT * C::kTileBytes;
    const uint32_t sO = sKV + C::kSlots * C::kTileBytes;  // 1024-aligned staging (NT == 2)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NT * C::kTileBytes + C::kSlots * C::kTileBytes +
                                                 C::kOStageBytes);
    float* stats = reinterpret_cast<float*>(bars + C::kNumBars);  // [2][NT][2][128]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(stats) + C::kStatsBytes);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const uint32_t bar0 = smem_u32(bars);
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (C::kSlots + s); };
    auto q_full = [&](int t) { return bar0 + 8u * (2 * C::kSlots + t); };
    auto q_empty = [&](int t) { return bar0 + 8u * (2 * C::kSlots + NT + t); };
    auto s_full = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 2 * NT + t); };
    auto p_full = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 3 * NT + t); };
    auto o_full = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 4 * NT + t); };
    auto o_empty = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 5 * NT + t); };
    // One barrier per statistics buffer: the softmax may post a unit's statistics before
    // the epilogue has waited for the previous unit's (a one-block unit's S needs nothing
    // from the epilogue), and a parity wait must never fall two phases behind.  Per buffer,
    // the next post needs the epilogue to have released O_t of the unit before.
    auto st_full = [&](int t, uint32_t buf) { return bar0 + 8u * (2 * C::kSlots + 6 * NT + 2 * t + buf); };
    const uint32_t mma_done = bar0 + 8u * (2 * C::kSlots + 8 * NT);
    // never arrived on: the injected stall waits on it (failure-detection tests)
    const uint32_t stall_bar = bar0 + 8u * (2 * C::kSlots + 8 * NT + 1);
    // separate P (kSepP): S_t read into registers (softmax -> MMA), P_t.V done (MMA -> softmax)
    [[maybe_unused]] auto s_free = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 8 * NT + 2 + t); };
    [[maybe_unused]] auto p_free = [&](int t) { return bar0 + 8u * (2 * C::kSlots + 8 * NT + 2 + NT + t); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
        }
        for (int t = 0; t < NT; ++t) {
            mbar_init(q_full(t), 1);
            mbar_init(q_empty(t), 1);
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), 128);
            mbar_init(o_full(t), 1);
            mbar_init(o_empty(t), 128);
            mbar_init(st_full(t, 0), 128);
            mbar_init(st_full(t, 1), 128);
        }
        mbar_init(mma_done, 1);
        mbar_init(stall_bar, 1);
        if constexpr (C::kSepP) {
            for (int t = 0; t < NT; ++t) {
                mbar_init(s_free(t), 128);
                mbar_init(p_free(t), 1);
            }
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
    }
    if (warp == 1) {
        tmem_alloc<C::kTmemCols>(smem_u32(tmem_slot));
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (wg == 0) {
        regs_dec<C::kRegsLoad>();
        if (warp == 0) {
            // -------------------------------------------------------- TMA producer
            // The whole warp runs the loop (so its values stay warp-uniform); one elected
            // lane issues the copies.
            uint32_t ld = 0;       // K/V ring loads issued (K and V each count one)
            uint32_t qn[NT] = {};  // Q loads issued per tile
            bool ok = true;
            PageCache pcache;      // paged KV only
            // Q_t of a unit, once the previous unit's last S_t has read the buffer
            auto load_q = [&](const UnitGeom<NT>& g, int t) {
                if (g.n[t] == 0 || !ok) return;
                if (qn[t] > 0)
                    ok = __all_sync(0xffffffffu, wait_bounded(q_empty(t), (qn[t] - 1) & 1u, abort_flag, p));
                if (!ok) return;
                if (elect_one()) {
                    const int rows = p.pack ? p.rows_valid : kBlockM;
                    mbar_arrive_expect_tx(q_full(t), (uint32_t)(rows * C::kRowBytes));
                    const int hcoord = p.pack ? g.hg * p.g : g.hg;
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_4d_hint(sQ + t * C::kTileBytes + c * C::kChunkBytes, &p.tm_q,
                                         q_full(t), c * 64, hcoord, g.pos0[t], g.b,
                                         l2_policy_evict_first());
                }
                __syncwarp();
                ++qn[t];
            };
            // Injected stall (failure-detection tests): a wait that nothing completes runs
            // out at the wait limit and aborts the CTA, as a copy that never lands would.
            if (p.inject_stall) ok = __all_sync(0xffffffffu, wait_bounded(stall_bar, 0u, abort_flag, p));
            // Load order per unit: Q_0, K_0, Q_1.., V_0, K_1, V_1, ...  The MMA warp may
            // issue a unit's first S_0 while the unit before still runs on tile 1, so K_0
            // must not queue behind Q_1 (which waits for that unit's last S_1).
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                const UnitGeom<NT> g = unit_geom<NT>(u, p);
                load_q(g, 0);
                for (int it = 0; it < g.nblk && ok; ++it) {
                    const int kpos = (g.kb_lo + it) * kBlockN;
                    // paged KV: the block's 128 keys come from 128 / page_rows pages (one
                    // page row range each); sub-ranges at or past this sequence's key count
                    // take a page coordinate past the pool, which TMA fills with zeros
                    // (masked anyway), so no table entry past the sequence is used
                    [[maybe_unused]] int pg[8], prow[8];
                    [[maybe_unused]] const int nsub = PAGED ? kBlockN / p.page_rows : 1;
                    if constexpr (PAGED) {
#pragma unroll
                        for (int sub = 0; sub < 8; ++sub) {
                            if (sub >= nsub) break;
                            const int key0 = kpos + sub * p.page_rows;
                            const int page = page_of(pcache, p, g.b, key0 >> p.page_shift, lane);
                            pg[sub] = key0 < g.sk ? page : p.num_pages;
                            prow[sub] = key0 & ((1 << p.page_shift) - 1);
                        }
                    }
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const int slot = ld % C::kSlots;
                        if (ld >= (uint32_t)C::kSlots)
                            ok = __all_sync(0xffffffffu, wait_bounded(kv_empty(slot), ((ld / C::kSlots) - 1) & 1u, abort_flag, p));
                        if (!ok) break;
                        if (elect_one()) {
                            mbar_arrive_expect_tx(kv_full(slot), (uint32_t)C::kTileBytes);
                            const void* tm = w == 0 ? (const void*)&p.tm_k : (const void*)&p.tm_v;
                            const uint64_t pol = p.kv_shared ? l2_policy_evict_last() : l2_policy_evict_first();
                            if constexpr (!PAGED) {
#pragma unroll
                                for (int c = 0; c < C::kChunks; ++c)
                                    tma_load_4d_hint(sKV + slot * C::kTileBytes + c * C::kChunkBytes, tm,
                                                     kv_full(slot), c * 64, g.kvh, kpos, g.b, pol);
                            } else {
#pragma unroll
                                for (int sub = 0; sub < 8; ++sub) {
                                    if (sub >= nsub) break;
#pragma unroll
                                    for (int c = 0; c < C::kChunks; ++c)
                                        tma_load_4d_hint(sKV + slot * C::kTileBytes + c * C::kChunkBytes +
                                                             sub * p.page_rows * C::kChunkRowBytes,
                                                         tm, kv_full(slot), c * 64, g.kvh, prow[sub],
                                                         pg[sub], pol);
                                }
                            }
                        }
                        __syncwarp();
                        ++ld;
                        if (it == 0 && w == 0) {
#pragma unroll
                            for (int t = 1; t < NT; ++t) load_q(g, t);
                        }
                    }
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA's memory is released
                const uint32_t first = ld > (uint32_t)C::kSlots ? ld - C::kSlots : 0u;
                for (uint32_t l = first; l < ld; ++l)
                    wait_drain(kv_full(l % C::kSlots), (l / C::kSlots) & 1u, p);
                for (int t = 0; t < NT; ++t)
                    if (qn[t] > 0) wait_drain(q_full(t), (qn[t] - 1) & 1u, p);
            }
            __syncwarp();
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer
            // The whole warp runs the loop: barrier waits and descriptors are warp-uniform,
            // and one elected lane issues each group of MMAs and its commit.
            uint32_t ld = 0;
            uint32_t qn[NT] = {}, pn[NT] = {}, on[NT] = {};
            bool ok = true;
            // descriptors built once; each MMA advances them by a constant offset
            const uint64_t q_desc0 = C::sdesc(sQ, 16);
            const uint64_t k_desc0 = C::sdesc(sKV, 16);
            const uint64_t v_desc0 = C::sdesc(sKV, C::kChunkBytes);  // MN-major: chunks along d
            // Issue a group of MMAs; before its last MMA, probe (without blocking) the
            // barrier the next group will wait on, so the probe's latency overlaps that
            // MMA instead of leaving the tensor pipe idle.  Returns the probe's result.
            auto issue_s = [&](int t, int slot, uint32_t probe_bar, uint32_t probe_par) {
                const uint64_t a0 = sdesc_add(q_desc0, t * C::kTileBytes);
                const uint64_t b0 = sdesc_add(k_desc0, slot * C::kTileBytes);
                const uint32_t d = tmem + C::s_col(t);
                bool ready = false;
                if (elect_one()) {
                    // 32 bytes of the row per MMA: 16 bf16 or 32 e4m3 of d
                    constexpr int kSteps = C::kRowBytes / 32;
#pragma unroll
                    for (int kk = 0; kk < kSteps; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                        if (kk == kSteps - 1 && probe_bar != 0u) ready = mbar_test_wait(probe_bar, probe_par);
                        C::mma_s(d, sdesc_add(a0, off), sdesc_add(b0, off), kk > 0 ? 1u : 0u);
                    }
                }
                return __ballot_sync(0xffffffffu, ready) != 0u;  // only the issuing lane probed
            };
            // O_t += P_t V over the block's 128 keys
            auto issue_pv = [&](int t, int slot, bool accumulate, uint32_t probe_bar,
                                uint32_t probe_par) {
                const uint64_t b0 = sdesc_add(v_desc0, slot * C::kTileBytes);
                const uint32_t d = tmem + C::o_col(t);
                const uint32_t a = tmem + C::p_col(t);
                bool ready = false;
                if (elect_one()) {
                    // 8 TMEM columns of P per MMA (16 bf16 or 32 e4m3 keys)
#pragma unroll
                    for (int kk = 0; kk < C::kPvSteps; ++kk) {
                        if (kk == C::kPvSteps - 1 && probe_bar != 0u) ready = mbar_test_wait(probe_bar, probe_par);
                        C::mma_pv(d, a + kk * 8, sdesc_add(b0, kk * C::kPvStepBytes),
                                  (accumulate || kk > 0) ? 1u : 0u);
                    }
                }
                return __ballot_sync(0xffffffffu, ready) != 0u;  // only the issuing lane probed
            };
            auto commit = [&](uint32_t bar) {
                if (elect_one()) mma_commit(bar);
                __syncwarp();
            };
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, p));
            };

            if constexpr (C::kSepP) {
            // Separate P: per key block, first S of the next block for every tile (once its
            // softmax has taken this block's S into registers), then P.V of this block.
            uint32_t sf[NT] = {};
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                const UnitGeom<NT> g = unit_geom<NT>(u, p);
                if (g.nblk == 0) continue;
                int slot_k = ld % C::kSlots;
                ok = wait(kv_full(slot_k), (ld / C::kSlots) & 1u);
                if (!ok) break;
                ++ld;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (g.n[t] == 0 || !ok) continue;
                    ok = wait(q_full(t), qn[t] & 1u);
                    if (!ok) break;
                    ++qn[t];
                    tc_fence_after();
                    issue_s(t, slot_k, 0u, 0u);
                    commit(s_full(t));
                    if (g.n[t] == 1) commit(q_empty(t));
                }
                if (!ok) break;
                commit(kv_empty(slot_k));
                for (int it = 0; it < g.nblk && ok; ++it) {
                    const int slot_v = ld % C::kSlots;
                    ok = wait(kv_full(slot_v), (ld / C::kSlots) & 1u);
                    if (!ok) break;
                    ++ld;
                    if (it + 1 < g.nblk) {
                        const int slot_n = ld % C::kSlots;
                        ok = wait(kv_full(slot_n), (ld / C::kSlots) & 1u);
                        if (!ok) break;
                        ++ld;
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            if (it + 1 >= g.n[t] || !ok) continue;
                            ok = wait(s_free(t), sf[t] & 1u);
                            if (!ok) break;
                            ++sf[t];
                            tc_fence_after();
                            issue_s(t, slot_n, 0u, 0u);
                            commit(s_full(t));
                            if (it + 2 == g.n[t]) commit(q_empty(t));
                        }
                        if (!ok) break;
                        commit(kv_empty(slot_n));
                    }
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (it >= g.n[t] || !ok) continue;
                        ok = wait(p_full(t), pn[t] & 1u);
                        if (!ok) break;
                        ++pn[t];
                        if (it == 0 && on[t] > 0) {
                            // the previous unit's epilogue must have read O_t out
                            ok = wait(o_empty(t), (on[t] - 1) & 1u);
                            if (!ok) break;
                        }
                        tc_fence_after();
                        issue_pv(t, slot_v, it > 0, 0u, 0u);
                        commit(p_free(t));
                        if (it + 1 == g.n[t]) {
                            commit(o_full(t));
                            ++on[t];
                        }
                    }
                    if (!ok) break;
                    commit(kv_empty(slot_v));
                }
            }
            } else {
            // A tile that finishes its unit starts the next unit at once: its first S_t is
            // issued right after its last PV_t (the tensor pipe runs MMAs in issue order,
            // so S_t may overwrite the P_t that PV_t reads), instead of after every tile's
            // last PV.  early[t]: the current unit's first S_t was issued that way.
            bool early[NT] = {};
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                const UnitGeom<NT> g = unit_geom<NT>(u, p);
                // key blocks per tile of the next unit (0 when there is none)
                int n_next[NT] = {};
                if (u + (int)gridDim.x < p.n_units) {
                    const UnitGeom<NT> gn = unit_geom<NT>(u + (int)gridDim.x, p);
#pragma unroll
                    for (int t = 0; t < NT; ++t) n_next[t] = gn.n[t];
                }
                bool early_next[NT] = {};
                if (g.nblk == 0) continue;
                // first key block: S_t for every tile that has keys (and was not started)
                const uint32_t ld_unit = ld;  // ring index of this unit's first K block
                int slot_k = ld % C::kSlots;
                ok = wait(kv_full(slot_k), (ld / C::kSlots) & 1u);
                if (!ok) break;
                ++ld;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (g.n[t] == 0 || early[t] || !ok) continue;
                    ok = wait(q_full(t), qn[t] & 1u);
                    if (!ok) break;
                    ++qn[t];
                    tc_fence_after();
                    issue_s(t, slot_k, 0u, 0u);
                    commit(s_full(t));
                    if (g.n[t] == 1) commit(q_empty(t));
                }
                if (!ok) break;
                commit(kv_empty(slot_k));

                bool v_ready = false;  // the next V block's barrier was already seen complete
                for (int it = 0; it < g.nblk && ok; ++it) {
                    const int slot_v = ld % C::kSlots;
                    if (!v_ready) ok = wait(kv_full(slot_v), (ld / C::kSlots) & 1u);
                    if (!ok) break;
                    ++ld;
                    // K of the next block: waited for only when its first S is issued
                    const bool next = it + 1 < g.nblk;
                    const uint32_t ld_n = ld;
                    const int slot_n = ld_n % C::kSlots;
                    const uint32_t kbar = kv_full(slot_n), kpar = (ld_n / C::kSlots) & 1u;
                    bool k_ready = false;
                    if (next) ++ld;
                    // the V block after next: probed at the end of this iteration
                    const uint32_t vbar = next ? kv_full(ld % C::kSlots) : 0u;
                    const uint32_t vpar = (ld / C::kSlots) & 1u;
                    v_ready = false;
                    tc_fence_after();
                    bool p_ready = false;  // this tile's P was already seen complete
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (it >= g.n[t] || !ok) continue;
                        if (!p_ready) ok = wait(p_full(t), pn[t] & 1u);
                        if (!ok) break;
                        ++pn[t];
                        if (it == 0 && on[t] > 0) {
                            // the previous unit's epilogue must have read O_t out
                            ok = wait(o_empty(t), (on[t] - 1) & 1u);
                            if (!ok) break;
                        }
                        tc_fence_after();
                        const bool more = it + 1 < g.n[t];
                        // probe what comes next: this tile's next K, else the next tile's P
                        const bool has_next_tile = (t + 1 < NT) && (it < g.n[t + 1 < NT ? t + 1 : t]);
                        const uint32_t pbar_next = has_next_tile ? p_full(t + 1 < NT ? t + 1 : t) : 0u;
                        const uint32_t ppar_next = has_next_tile ? (pn[t + 1 < NT ? t + 1 : t] & 1u) : 0u;
                        bool probed = issue_pv(t, slot_v, it > 0,
                                               more && !k_ready ? kbar : pbar_next,
                                               more && !k_ready ? kpar : ppar_next);
                        if (more) {
                            if (!k_ready) {
                                if (!probed) ok = wait(kbar, kpar);
                                if (!ok) break;
                                k_ready = true;
                                tc_fence_after();
                            }
                            p_ready = issue_s(t, slot_n, has_next_tile ? pbar_next : vbar,
                                              has_next_tile ? ppar_next : vpar);
                            if (!has_next_tile) {
                                v_ready = p_ready;
                                p_ready = false;
                            }
                            commit(s_full(t));
                            if (it + 2 == g.n[t]) commit(q_empty(t));
                        } else {
                            p_ready = has_next_tile && probed;
                            commit(o_full(t));
                            ++on[t];
                            // The next unit's K_0 sits at ring index ld_unit + 2 nblk.  Taking
                            // it now is safe when the ring entry it replaces was consumed and
                            // released by an earlier iteration (or the prologue): then its
                            // barrier phase is current and the producer is not blocked on
                            // anything issued later.
                            if (n_next[t] > 0 && 2 * (g.nblk - it) <= C::kSlots) {
                                const uint32_t kq = ld_unit + 2u * (uint32_t)g.nblk;
                                ok = wait(kv_full(kq % C::kSlots), (kq / C::kSlots) & 1u);
                                if (ok) ok = wait(q_full(t), qn[t] & 1u);
                                if (!ok) break;
                                ++qn[t];
                                tc_fence_after();
                                issue_s(t, kq % C::kSlots, 0u, 0u);
                                commit(s_full(t));
                                if (n_next[t] == 1) commit(q_empty(t));
                                early_next[t] = true;
                            }
                        }
                    }
                    if (!ok) break;
                    commit(kv_empty(slot_v));
                    if (next) commit(kv_empty(slot_n));
                }
#pragma unroll
                for (int t = 0; t < NT; ++t) early[t] = early_next[t];
            }
            }
            // every MMA issued so far must be complete before TMEM is released
            commit(mma_done);
            wait_drain(mma_done, 0u, p);
            __syncwarp();
        }
    } else if (wg <= NT) {
        // ------------------------------------------------------------ softmax, tile t
        regs_inc<C::kRegsSoftmax>();
        const int t = wg - 1;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t s_addr = tmem + ((uint32_t)(quarter * 32) << 16) + C::s_col(t);
        const uint32_t o_addr = tmem + ((uint32_t)(quarter * 32) << 16) + C::o_col(t);
        static_assert(!C::kSepP || (C::p_col(0) - C::o_col(0) == C::kPAfterO &&
                                    C::p_col(NT - 1) - C::o_col(NT - 1) == C::kPAfterO),
                      "separate P lies a fixed distance past O");
        // P's columns: S's own, or (separate P) a fixed distance past O's
        const uint32_t p_addr = C::kSepP ? o_addr + C::kPAfterO : s_addr;
        const float c = p.scale_log2;
        const float kNegInf = -INFINITY;
        const float fill = (c >= 0.f) ? -INFINITY : INFINITY;  // masked keys drop out of the extremum
        uint32_t sn = 0, stn = 0, sn_o = 0;
        bool ok = true;

        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
            const UnitGeom<NT> g = unit_geom<NT>(u, p);
            const int n_t = pick<NT>(g.n, t);
            const RowMap rm = row_map(p, pick<NT>(g.pos0, t), g.hg, row);
            if (n_t == 0) {
                if constexpr (!C::kEpilogueWG)
                    write_row<HD>(p, o_addr, rm, g.b, g.split, false, true, -INFINITY, 0.f, 0u);
                continue;
            }
            // exclusive key bound of this row (causal: j <= pos + Sk - Sq)
            const int kmax = p.causal ? min(g.sk, rm.pos + 1 + (g.sk - p.Sq)) : g.sk;
            // A warp whose 32 rows are all padding (short query axis, e.g. decode) only
            // keeps the handshake: its P and O rows feed nothing that is stored.
            const bool idle = __all_sync(0xffffffffu, !rm.ok);
            if (idle) {
                for (int it = 0; it < n_t && ok; ++it) {
                    ok = __all_sync(0xffffffffu, wait_bounded(s_full(t), sn & 1u, abort_flag, p));
                    if (!ok) break;
                    ++sn;
                    tc_fence_after();
                    tc_fence_before();
                    if constexpr (C::kSepP) {
                        if (it + 1 < n_t) mbar_arrive(s_free(t));
                        // The next S may already be issued, so this warp could reach the
                        // next block before the others finish this block's P: its early
                        // arrivals would then complete this block's p_full.  Waiting for
                        // the previous P.V keeps one arrival per thread per phase.
                        // sn - 1 blocks of this tile came before this one
                        if (sn > 1) {
                            ok = __all_sync(0xffffffffu, wait_bounded(p_free(t), sn & 1u, abort_flag, p));
                            if (!ok) break;
                        }
                    }
                    mbar_arrive(p_full(t));
                }
                if (!ok) break;
                if constexpr (C::kEpilogueWG) {
                    mbar_arrive(st_full(t, stn & 1u));
                    ++stn;
                } else {
                    ok = __all_sync(0xffffffffu, wait_bounded(o_full(t), sn_o & 1u, abort_flag, p));
                    if (!ok) break;
                    ++sn_o;
                    tc_fence_after();
                    write_row<HD>(p, o_addr, rm, g.b, g.split, true, true, kNegInf, 0.f, o_empty(t));
                }
                continue;
            }

            float m = 0.f;  // reference max of c*s (log2 units), see below
            float l = 0.f;
            for (int it = 0; it < n_t; ++it) {
                ok = __all_sync(0xffffffffu, wait_bounded(s_full(t), sn & 1u, abort_flag, p));
                if (!ok) break;
                ++sn;
                tc_fence_after();
                float s[128];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t r[32];
                    tmem_ld32(s_addr + ch * 32, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[ch * 32 + i] = __uint_as_float(r[i]);
                }
                tmem_wait_ld();
                if constexpr (C::kSepP) {
                    // S is in registers: the next block's S may be written over it
                    if (it + 1 < n_t) {
                        tc_fence_before();
                        mbar_arrive(s_free(t));
                    }
                }
                const int lim = kmax - (g.kb_lo + it) * kBlockN;  // keys [0, lim) allowed
                // Warp-uniform view of the mask, per 32-key chunk: every key allowed for all
                // 32 rows of the warp (full), none allowed for any of them (empty), or in
                // between.  The branches on it are uniform, as the warp-collective tcgen05.st
                // in the exponential loop requires.  Unmasked blocks skip all of it.
                const int lim_lo = __reduce_min_sync(0xffffffffu, lim);
                const int lim_hi = __reduce_max_sync(0xffffffffu, lim);
                const bool masked = lim_lo < kBlockN;
                auto chunk_empty = [&](int ch) { return ch * 32 >= lim_hi; };
                auto chunk_full = [&](int ch) { return ch * 32 + 32 <= lim_lo; };
                // extremum of the raw scores over the allowed keys (max for c >= 0, min for
                // c < 0); disallowed keys of a partial chunk take the fill value first
                auto extremum = [&](auto op3, auto op2) -> float {
                    if (!masked) {
                        float e[8];  // eight chains of three-input max/min
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            e[k] = op3(s[k], s[k + 8], s[k + 16]);
#pragma unroll
                            for (int i = 3; i < 15; i += 2) e[k] = op3(e[k], s[k + 8 * i], s[k + 8 * i + 8]);
                            e[k] = op2(e[k], s[k + 120]);
                        }
                        return op2(op3(e[0], e[1], e[2]), op3(e[3], e[4], op3(e[5], e[6], e[7])));
                    }
                    float acc = fill;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        if (chunk_empty(ch)) continue;
                        const int b0 = ch * 32;
                        if (!chunk_full(ch)) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) s[b0 + i] = (b0 + i < lim) ? s[b0 + i] : fill;
                        }
                        float e[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            e[k] = op3(s[b0 + k], s[b0 + k + 4], s[b0 + k + 8]);
                            e[k] = op3(e[k], s[b0 + k + 12], s[b0 + k + 16]);
                            e[k] = op3(e[k], s[b0 + k + 20], s[b0 + k + 24]);
                            e[k] = op2(e[k], s[b0 + k + 28]);
                        }
                        acc = op3(acc, op3(e[0], e[1], e[2]), e[3]);
                    }
                    return acc;
                };
                float e[1];
                if (c >= 0.f)
                    e[0] = extremum([](float x, float y, float z) { return max3(x, y, z); },
                                    [](float x, float y) { return fmaxf(x, y); });
                else
                    e[0] = extremum([](float x, float y, float z) { return min3(x, y, z); },
                                    [](float x, float y) { return fminf(x, y); });
                const float mx = (lim <= 0) ? kNegInf : (c == 0.f ? 0.f : e[0] * c);
                // Reference max m (log2 units).  It starts at 0, not at the row's first
                // block max, and moves only when a block's max leaves the window [m - 64,
                // m + 8]: up past m + 8 (deferred rescaling, which keeps every p <= 256),
                // or, while nothing has been summed yet, far below m (keys whose p would
                // underflow).  It then moves to the block max rounded up to an integer.
                // For scores within the window (typical attention logits) m stays 0 in every
                // schedule, so x = c s is rounded once, the same way whether the key axis is
                // split or the heads packed, and P is bit-identical across the scheduling
                // variants; where m does move, it moves by integers, so p changes by exact
                // powers of two and the rescale factors are exact.  With e4m3 P, whose
                // smallest value is 2^-9 and whose normals start at 2^-6, the lower edge is
                // m - 1 and a move leaves the block max 4 octaves above m (p_max in (8, 16]):
                // the row's largest p is then always >= 1/2 (m <= the row max + 1), and keys
                // up to 9 octaves below the max keep e4m3's full 3-bit precision.  Moves are
                // still by integers, and e4m3 rounding commutes with powers of two.
                constexpr float kLowEdge = F8 ? 1.0f : 64.f;
                constexpr float kHeadroom = F8 ? 4.0f : 0.f;
                const bool grow = mx > m + 8.0f || (l == 0.f && mx > kNegInf && mx < m - kLowEdge);
                float alpha = 1.f;
                if (grow) {
                    const float m_new = ceilf(mx) - kHeadroom;
                    alpha = (l == 0.f) ? 0.f : ex2_approx(m - m_new);  // nothing summed: O is 0
                    l *= alpha;
                    m = m_new;
                }
                // P = 2^(c*s - m) as bf16, written over S in TMEM (S is in registers).  A
                // disallowed key gets the exponent -inf, i.e. p = 0, for any sign of c.
                const float neg_m = -m;
                float ls0 = 0.f, ls1 = 0.f;
                // the pairs of a chunk that take the polynomial, spread over the chunk
                auto use_poly = [](int ch, int i) { return ((i * 5 + ch * 3) & 15) < C::kPolyPairs; };
                // P of 32-key chunk ch into TMEM over S: 16 columns of bf16 pairs, or 8 of e4m3
                // quads (pk[0..7])
                auto store_p = [&](int ch, const uint32_t (&pk)[16]) {
                    if constexpr (F8) {
                        uint32_t q8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) q8[i] = pk[i];
                        tmem_st8(p_addr + ch * C::kPColsPer32, q8);
                    } else {
                        tmem_st16(p_addr + ch * C::kPColsPer32, pk);
                    }
                };
                // one 32-key chunk: P = 2^(c s - m) as bf16 pairs; with kSelect, keys at or
                // past lim get the exponent -inf (p = 0 for either sign of c)
                auto exp_chunk = [&](auto select_c, int ch) {
                    constexpr bool kSelect = decltype(select_c)::value;
                    uint32_t pk[16];  // P of the chunk: 16 bf16 pairs, or 8 e4m3 quads
                    [[maybe_unused]] float p_even0 = 0.f, p_even1 = 0.f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int j = ch * 32 + 2 * i;
                        float x0, x1, p0, p1;
                        fma2(s[j], s[j + 1], c, c, neg_m, neg_m, x0, x1);
                        if constexpr (kSelect) {
                            x0 = (j < lim) ? x0 : kNegInf;
                            x1 = (j + 1 < lim) ? x1 : kNegInf;
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        } else if (use_poly(ch, i)) {
                            exp2_poly2(x0, x1, p0, p1);
                        } else {
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        add2(ls0, ls1, p0, p1, ls0, ls1);
                        if constexpr (F8) {
                            if (i & 1) pk[i >> 1] = pack_e4m3x4(p_even0, p_even1, p0, p1);
                            else {
                                p_even0 = p0;
                                p_even1 = p1;
                            }
                        } else {
                            pk[i] = pack_bf16x2(p0, p1);
                        }
                    }
                    store_p(ch, pk);
                };
                auto exp_range = [&](auto masked_c, int ch0, int ch1) {
                    constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
                    for (int ch = ch0; ch < ch1; ++ch) {
                        if (!kMasked || chunk_full(ch)) {
                            exp_chunk(std::false_type{}, ch);
                        } else if (chunk_empty(ch)) {
                            uint32_t pk[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) pk[i] = 0u;  // zeros in either format
                            store_p(ch, pk);
                        } else {
                            exp_chunk(std::true_type{}, ch);
                        }
                    }
                };
                if constexpr (C::kSepP) {
                    // the previous block's P.V must be done before P and O are written again
                    // P.V of block sn - 2 (this tile's previous one, if any)
                    if (sn > 1) {
                        ok = __all_sync(0xffffffffu, wait_bounded(p_free(t), sn & 1u, abort_flag, p));
                        if (!ok) break;
                        tc_fence_after();
                    }
                }
                if (masked) exp_range(std::true_type{}, 0, 2);
                else exp_range(std::false_type{}, 0, 2);
                // O rescale: PV of the previous block is complete, because this block's S
                // was issued after it.
                if (it > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
                    for (int ch = 0; ch < HD / 32; ++ch) {
                        uint32_t r[32];
                        tmem_ld32(o_addr + ch * 32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tmem_st32(o_addr + ch * 32, r);
                    }
                }
                // second half: keys 64..127
                if (masked) exp_range(std::true_type{}, 2, 4);
                else exp_range(std::false_type{}, 2, 4);
                l += ls0 + ls1;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full(t));
            }
            if (!ok) break;
            if constexpr (C::kEpilogueWG) {
                // row statistics for the epilogue warpgroup (double-buffered by unit)
                float* st = stats + ((stn & 1u) * NT + t) * 256;
                st[row] = m;
                st[128 + row] = l;
                mbar_arrive(st_full(t, stn & 1u));
                ++stn;
            } else {
                ok = __all_sync(0xffffffffu, wait_bounded(o_full(t), sn_o & 1u, abort_flag, p));
                if (!ok) break;
                ++sn_o;
                tc_fence_after();
                write_row<HD>(p, o_addr, rm, g.b, g.split, true, false, m, l, o_empty(t));
            }
        }
    } else if constexpr (C::kEpilogueWG) {
        // ------------------------------------------------------------ epilogue
        // O / l goes out through a swizzled shared-memory stage and TMA tensor stores, a
        // 32-column chunk at a time, so every global write is a full line; LSE is stored
        // directly.
        if constexpr (C::kRegsEpilogue < C::kLaunchRegs) regs_dec<C::kRegsEpilogue>();
        if constexpr (C::kRegsEpilogue > C::kLaunchRegs) regs_inc<C::kRegsEpilogue>();
        constexpr uint32_t kEpiBar = 1;  // named barrier of the four epilogue warps
        constexpr float kLn2 = 0.69314718055994530942f;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const bool issuer = (threadIdx.x == (1 + NT) * 128);
        uint32_t on[NT] = {}, stn[NT] = {};
        bool ok = true;
        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
            const UnitGeom<NT> g = unit_geom<NT>(u, p);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (!ok) break;
                if (g.pos0[t] >= p.Sq) continue;  // a tile wholly past the query axis (uniform)
                const RowMap rm = row_map(p, g.pos0[t], g.hg, row);
                const bool has = g.n[t] > 0;
                const bool idle = __all_sync(0xffffffffu, !rm.ok);
                float m = -INFINITY, l = 0.f;
                if (has) {
                    ok = __all_sync(0xffffffffu, wait_bounded(st_full(t, stn[t] & 1u), (stn[t] >> 1) & 1u,
                                                              abort_flag, p));
                    if (ok) {
                        const float* st = stats + ((stn[t] & 1u) * NT + t) * 256;
                        m = st[row];
                        l = st[128 + row];
                        ++stn[t];
                        ok = __all_sync(0xffffffffu, wait_bounded(o_full(t), on[t] & 1u, abort_flag, p));
                        ++on[t];
                    }
                }
                // one decision for the whole warpgroup before its named barriers
                ok = named_bar_and(kEpiBar, 128, ok);
                if (!ok) break;
                tc_fence_after();
                const float inv_l = (l > 0.f) ? p.v_scale / l : 0.f;
                const float lse_v = (l > 0.f) ? (m + __log2f(l)) * kLn2 : -INFINITY;
                const uint32_t o_addr = tmem + ((uint32_t)(quarter * 32) << 16) + C::o_col(t);
                const int hcoord = p.pack ? g.hg * p.g : g.hg;
                const int bcoord = p.num_splits == 1 ? g.b : g.split * p.B + g.b;
                // bf16 output (final output only): a stage row holds 64 bf16 columns, filled
                // from two 32-column TMEM chunks, then one TMA store of 64 columns
                const bool bf16_out = p.out_bf16 != nullptr && p.num_splits == 1;
                if (bf16_out) {
#pragma unroll
                    for (int ch = 0; ch < HD / 32; ++ch) {
                        uint32_t r[32];
                        if (has && !idle) {
                            tmem_ld32(o_addr + ch * 32, r);
                            tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) r[i] = 0u;
                        }
                        if (has && ch == HD / 32 - 1) {
                            tc_fence_before();
                            mbar_arrive(o_empty(t));
                        }
                        const int half = ch & 1;
                        if (half == 0) {
                            if (issuer) bulk_wait_read_all();
                            named_bar_sync(kEpiBar, 128);
                        }
                        const uint32_t dst = sO + row * 128;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t a = dst + ((uint32_t)((half * 4 + j) ^ (row & 7)) << 4);
                            const float* f = reinterpret_cast<const float*>(r) + 8 * j;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                                         "r"(pack_bf16x2(f[0] * inv_l, f[1] * inv_l)),
                                         "r"(pack_bf16x2(f[2] * inv_l, f[3] * inv_l)),
                                         "r"(pack_bf16x2(f[4] * inv_l, f[5] * inv_l)),
                                         "r"(pack_bf16x2(f[6] * inv_l, f[7] * inv_l))
                                         : "memory");
                        }
                        if (half == 1) {
                            fence_proxy_async_smem();
                            named_bar_sync(kEpiBar, 128);
                            if (issuer) {
                                tma_store_4d_hint(&p.tm_o, sO, (ch >> 1) * 64, hcoord, g.pos0[t], bcoord,
                                                  l2_policy_evict_first());
                                bulk_commit_group();
                            }
                        }
                    }
                } else {
#pragma unroll
                for (int ch = 0; ch < HD / 32; ++ch) {
                    uint32_t r[32];
                    if (has && !idle) {
                        tmem_ld32(o_addr + ch * 32, r);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = 0u;
                    }
                    if (has && ch == HD / 32 - 1) {
                        // O_t is in registers: the next unit's PV may overwrite it
                        tc_fence_before();
                        mbar_arrive(o_empty(t));
                    }
                    // the stage is free once the previous store has read it
                    if (issuer) bulk_wait_read_all();
                    named_bar_sync(kEpiBar, 128);
                    const uint32_t dst = sO + row * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t a = dst + ((uint32_t)(i ^ (row & 7)) << 4);
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                                     "f"(__uint_as_float(r[4 * i + 0]) * inv_l),
                                     "f"(__uint_as_float(r[4 * i + 1]) * inv_l),
                                     "f"(__uint_as_float(r[4 * i + 2]) * inv_l),
                                     "f"(__uint_as_float(r[4 * i + 3]) * inv_l)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(kEpiBar, 128);
                    if (issuer) {
                        // the final output is not read again here; split partials are,
                        // by the combine, and keep the default policy
                        if (p.num_splits == 1)
                            tma_store_4d_hint(&p.tm_o, sO, ch * 32, hcoord, g.pos0[t], bcoord,
                                              l2_policy_evict_first());
                        else
                            tma_store_4d(&p.tm_o, sO, ch * 32, hcoord, g.pos0[t], bcoord);
                        bulk_commit_group();
                    }
                }
                }
                if (rm.ok) {
                    if (p.num_splits == 1)
                        p.lse[((size_t)g.b * p.Hq + rm.head) * p.Sq + rm.pos] = lse_v;
                    else
                        p.lse_part[(((size_t)g.split * p.B + g.b) * p.Hq + rm.head) * p.Sq + rm.pos] = lse_v;
                }
            }
        }
        if (issuer) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<C::kTmemCols>(tmem);
    }
}

// ---------------------------------------------------------------- unit order by work
// With per-sequence key lengths the units' work varies from nothing to the capacity; a
// static stride over them leaves the CTA that draws long sequences last.  This pre-pass
// (one CTA) sorts the units by their key-block count, heaviest first (a counting sort;
// counts above kBuckets - 1 share the top bucket), and deals them in rounds of `grid`
// positions, alternating direction (round r gives its k-th heaviest unit to CTA k when r is
// even, to CTA grid-1-k when r is odd; a last partial round goes in order).  order[u] is
// the unit that position u of the kernel's static stride takes.  sorted_tmp holds n_units
// entries.  The order only moves work between CTAs: every unit is still computed once.
template <int NT>
__global__ void __launch_bounds__(1024) gqa_unit_order_kernel(const __grid_constant__ FwdParams p,
                                                              int grid, int* order,
                                                              int* sorted_tmp) {
    constexpr int kBuckets = 2048;
    __shared__ int cnt[kBuckets];
    for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    FwdParams q = p;
    q.unit_order = nullptr;
    auto bucket_of = [&](int u) {
        const int n = unit_geom<NT>(u, q).nblk;
        return kBuckets - 1 - (n < kBuckets - 1 ? n : kBuckets - 1);  // heaviest first
    };
    for (int u = threadIdx.x; u < p.n_units; u += blockDim.x) atomicAdd(&cnt[bucket_of(u)], 1);
    __syncthreads();
    // exclusive prefix sum of the counts: each of the 1024 threads owns kPer consecutive
    // buckets; warp shuffles scan the threads' totals, one warp scans the warps' totals
    {
        constexpr int kPer = kBuckets / 1024;
        __shared__ int warp_sum[32];
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        int own[kPer];
        int tot = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            own[j] = cnt[threadIdx.x * kPer + j];
            tot += own[j];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sum[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        int base = incl - tot + (warp > 0 ? warp_sum[warp - 1] : 0);
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            cnt[threadIdx.x * kPer + j] = base;
            base += own[j];
        }
    }
    __syncthreads();
    for (int u = threadIdx.x; u < p.n_units; u += blockDim.x)
        sorted_tmp[atomicAdd(&cnt[bucket_of(u)], 1)] = u;
    __syncthreads();
    const int full_rounds = p.n_units / grid;
    for (int pos = threadIdx.x; pos < p.n_units; pos += blockDim.x) {
        const int r = pos / grid, k = pos - r * grid;
        const int src = (r < full_rounds && (r & 1)) ? r * grid + (grid - 1 - k) : pos;
        order[pos] = sorted_tmp[src];
    }
}

// ---------------------------------------------------------------- split-KV combine
// One warp per output row (b, h, i): M = max_s lse_s, w_s = exp(lse_s - M),
// lse = M + ln sum w_s, O = sum_s w_s O_s / sum_s w_s.
template <int HD>
__global__ void __launch_bounds__(256) gqa_combine_kernel(const CombineParams p) {
    constexpr int kPer = HD / 32;
    const long long rows = (long long)p.B * p.Hq * p.Sq;
    const int lane = threadIdx.x & 31;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    const float kNegInf = -INFINITY;
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps_total) {
        float ls = (lane < p.num_splits) ? p.lse_part[(long long)lane * rows + r] : kNegInf;
        float M = ls;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float w = (M == kNegInf || ls == kNegInf) ? 0.f : __expf(ls - M);
        float wsum = w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        float acc[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
        // r = (b * Hq + h) * Sq + i; partials are [split, B, Sq, Hq, d]
        const long long ii = r % p.Sq;
        const long long hh = (r / p.Sq) % p.Hq;
        const long long bb = r / ((long long)p.Sq * p.Hq);
        for (int s = 0; s < p.num_splits; ++s) {
            const float ws = __shfl_sync(0xffffffffu, w, s);
            if (ws == 0.f) continue;
            const float* src = p.o_part + ((((long long)s * p.B + bb) * p.Sq + ii) * p.Hq + hh) * HD + lane * kPer;
            if constexpr (kPer == 4) {
                const float4 v = *reinterpret_cast<const float4*>(src);
                acc[0] += ws * v.x;
                acc[1] += ws * v.y;
                acc[2] += ws * v.z;
                acc[3] += ws * v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(src);
                acc[0] += ws * v.x;
                acc[1] += ws * v.y;
            }
        }
        const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
        // r = (b * Hq + h) * Sq + i  ->  out[b, i, h, :]
        const long long i = r % p.Sq;
        const long long bh = r / p.Sq;
        const long long h = bh % p.Hq;
        const long long b = bh / p.Hq;
        const long long off = ((b * p.Sq + i) * p.Hq + h) * HD + lane * kPer;
        if (p.out_bf16 != nullptr) {
            uint16_t* dst = p.out_bf16 + off;
            if constexpr (kPer == 4) {
                *reinterpret_cast<uint2*>(dst) = make_uint2(ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                            ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv));
            } else {
                *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
            }
        } else {
            float* dst = p.out + off;
            if constexpr (kPer == 4) {
                *reinterpret_cast<float4*>(dst) =
                    make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
            } else {
                *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
            }
        }
        if (lane == 0) p.lse[r] = (wsum > 0.f) ? M + __logf(wsum) : kNegInf;
    }
}

template <int HD, int NT, bool F8, bool PAGED>
cudaError_t launch_fwd_t(const FwdParams& p, int grid, cudaStream_t stream) {
    using C = FwdCfg<HD, NT, F8>;
    // the attribute is per device; setting it again is idempotent, so the race is benign
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gqa_fwd_kernel<HD, NT, F8, PAGED>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    // setmaxnreg redistributes the registers the CTA was launched with: refuse to launch
    // a build whose register count differs from the split's assumption
    static int regs_checked = 0;  // 0 unknown, 1 ok, -1 mismatch
    if (regs_checked == 0) {
        cudaFuncAttributes attr{};
        cudaError_t e = cudaFuncGetAttributes(&attr, gqa_fwd_kernel<HD, NT, F8, PAGED>);
        if (e != cudaSuccess) return e;
        regs_checked = (attr.numRegs == C::kLaunchRegs) ? 1 : -1;
    }
    if (regs_checked != 1) return cudaErrorInvalidConfiguration;
    gqa_fwd_kernel<HD, NT, F8, PAGED><<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int fwd_ctas_per_sm(int hd, int nt) {
    if (nt == 2) return hd == 128 ? FwdCfg<128, 2>::kCtasPerSm : FwdCfg<64, 2>::kCtasPerSm;
    return hd == 128 ? FwdCfg<128, 1>::kCtasPerSm : FwdCfg<64, 1>::kCtasPerSm;
}

cudaError_t launch_fwd(const FwdParams& p, int hd, int nt, bool f8, int grid, cudaStream_t stream) {
    if (f8) {
        if (hd == 128) return nt == 2 ? launch_fwd_t<128, 2, true, false>(p, grid, stream) : launch_fwd_t<128, 1, true, false>(p, grid, stream);
        return nt == 2 ? launch_fwd_t<64, 2, true, false>(p, grid, stream) : launch_fwd_t<64, 1, true, false>(p, grid, stream);
    }
    if (p.block_table != nullptr) {
        if (hd == 128) return nt == 2 ? launch_fwd_t<128, 2, false, true>(p, grid, stream) : launch_fwd_t<128, 1, false, true>(p, grid, stream);
        return nt == 2 ? launch_fwd_t<64, 2, false, true>(p, grid, stream) : launch_fwd_t<64, 1, false, true>(p, grid, stream);
    }
    if (hd == 128) return nt == 2 ? launch_fwd_t<128, 2, false, false>(p, grid, stream) : launch_fwd_t<128, 1, false, false>(p, grid, stream);
    return nt == 2 ? launch_fwd_t<64, 2, false, false>(p, grid, stream) : launch_fwd_t<64, 1, false, false>(p, grid, stream);
}

cudaError_t launch_unit_order(const FwdParams& p, int nt, int grid, int* order, int* tmp,
                              cudaStream_t stream) {
    if (nt == 2)
        gqa_unit_order_kernel<2><<<1, 1024, 0, stream>>>(p, grid, order, tmp);
    else
        gqa_unit_order_kernel<1><<<1, 1024, 0, stream>>>(p, grid, order, tmp);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams& p, int hd, int num_sms, cudaStream_t stream) {
    const long long rows = (long long)p.B * p.Hq * p.Sq;
    long long blocks = (rows + 7) / 8;
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (hd == 128)
        gqa_combine_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else
        gqa_combine_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

unsigned int* device_status_symbol() {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) return nullptr;
    return static_cast<unsigned int*>(ptr);
}

}  // namespace gqa
