// C ABI of libgqa_attn.so: argument validation, the pack/split heuristic, TMA tensor
// maps, split-KV scratch and kernel launches.  See include/gqa_attn.h for the contract.
#include "gqa_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "fwd_params.h"
#include "launch.h"

namespace {

using gqa::kBlockM;
using gqa::kBlockN;
using gqa::kMaxSplits;

constexpr int kDefaultSms = 148;

struct Plan {
    int pack;        // 0 / 1
    int nt;          // tiles per CTA unit (1 or 2)
    int pos_per_tile;
    int rows_valid;
    int n_hg;
    int n_mt;
    int splits;      // resolved, clamped
    int kv_blocks;
    long long units;
};

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

gqa_status validate_shape(int B, int Sq, int Sk, int Hq, int Hk, int d, int pack, int splits) {
    if (B < 1 || Sq < 1 || Sk < 1 || Hq < 1 || Hk < 1) return GQA_ERR_SHAPE;
    if (pack < -1 || pack > 1 || splits < 0) return GQA_ERR_SHAPE;
    if (Hq % Hk != 0) return GQA_ERR_HEADS;
    if (d != 64 && d != 128) return GQA_ERR_HEADDIM;
    if (pack == 1 && Hq / Hk > kBlockM) return GQA_ERR_SHAPE;  // one position must fit a tile
    // TMA coordinates and in-kernel row indices are 32-bit
    const long long rows_out = (long long)B * Hq * Sq;
    if (rows_out >= (1ll << 31) || (long long)B * Sk * Hk >= (1ll << 31)) return GQA_ERR_SHAPE;
    return GQA_OK;
}

// Padded tile rows computed per kv group with and without packing.
void padded_rows(int Sq, int g, long long* unpacked, long long* packed) {
    *unpacked = (long long)g * ceil_div(Sq, kBlockM) * kBlockM;
    const int P = kBlockM / g;
    *packed = P >= 1 ? (long long)ceil_div(Sq, P) * kBlockM : (1ll << 62);
}

// Pack when it pads fewer tile rows.  Causal attention also packs at equal rows: a unit's
// two packed tiles cover adjacent short position ranges whose diagonals fall in the same
// key block, so both tiles finish on the same block, while two 128-position tiles end a
// block apart and the unit's last block runs one tile alone (measured on B200, causal:
// +6 % at B=64 S=2048, +16 % at S=1024, +15 % at d=64, within 1.5 % at S=16384).
int choose_pack(int Sq, int Hq, int Hk, int causal) {
    const int g = Hq / Hk;
    if (g == 1 || g > kBlockM) return 0;
    long long un, pk;
    padded_rows(Sq, g, &un, &pk);
    return (pk < un || (causal && pk == un)) ? 1 : 0;
}

// Fill everything except the split count from the shape and the pack choice.
Plan make_plan(int B, int Sq, int Sk, int Hq, int Hk, int pack) {
    Plan pl{};
    const int g = Hq / Hk;
    pl.pack = pack;
    pl.pos_per_tile = pack ? kBlockM / g : kBlockM;
    pl.rows_valid = pack ? g * pl.pos_per_tile : kBlockM;
    pl.n_hg = pack ? Hk : Hq;
    const int tiles = ceil_div(Sq, pl.pos_per_tile);
    pl.nt = tiles >= 2 ? 2 : 1;
    pl.n_mt = ceil_div(tiles, pl.nt);
    pl.kv_blocks = ceil_div(Sk, kBlockN);
    pl.units = (long long)pl.n_mt * B * pl.n_hg;
    (void)B;
    return pl;
}

// Split count minimising the modelled time: waves(s) x (key blocks per split + a fixed
// per-unit cost).  A persistent CTA per SM slot takes units in a static stride, so a
// partial last wave costs a whole unit time.  The fixed cost (Q load, pipeline fill,
// epilogue, and the partials' write and combine) was fitted to B200 measurements of
// the decode grid (Sk 2K-32K, B 32-256): about four key blocks' worth; a split must
// also buy at least 5 %, since the combine adds a launch.
int choose_splits(const Plan& pl, int d, int num_sms) {
    const long long slots = (long long)num_sms * gqa::fwd_ctas_per_sm(d, pl.nt);
    const int smax = pl.kv_blocks < kMaxSplits ? pl.kv_blocks : kMaxSplits;
    constexpr double kUnitCost = 4.0;
    int best = 1;
    double best_t = 0.0;
    for (int s = 1; s <= smax; ++s) {
        const long long waves = (pl.units * s + slots - 1) / slots;
        const double t = (double)waves * ((double)pl.kv_blocks / s + kUnitCost);
        if (s == 1 || t < best_t * 0.95) {
            best = s;
            best_t = t;
        }
    }
    return best;
}

// With per-sequence KV lengths the units' work varies from nothing to the capacity, and
// the plan cannot see the lengths (they live on the device).  Split until there are at
// least kVarlenUnitsPerSlot units per CTA slot: the device-side work order then deals
// them heaviest first over the CTAs (one-tile kernel), and a slot sums several units of
// unrelated length.  The prefill kernel keeps its own order, so it also takes at least
// the dense model's count for the capacity.
int choose_splits_varlen(const Plan& pl, int d, int num_sms) {
    constexpr long long kVarlenUnitsPerSlot = 3;  // fitted on B200: uniform lengths, B 32-256
    const long long slots = (long long)num_sms * gqa::fwd_ctas_per_sm(d, pl.nt);
    const int smax = pl.kv_blocks < kMaxSplits ? pl.kv_blocks : kMaxSplits;
    int s = 1;
    while (s < smax && pl.units * s < kVarlenUnitsPerSlot * slots) ++s;
    if (pl.nt == 1) return s;
    const int dense = choose_splits(pl, d, num_sms);
    return s > dense ? s : dense;
}

// Tuned schedules, read once per process from the text file named by GQA_TUNE_TABLE, or
// when that is unset from the table shipped beside the library (both as written by the
// package's autotune module).  One entry per line:
//   d causal Hq Hk bucket(B) bucket(Sq) bucket(Sk) pack_gqa num_splits [anything else]
// with bucket(x) = the smallest e such that 2^e >= x.  '#' starts a comment line; lines
// that do not parse are skipped; a later line for the same key wins.
struct TuneEntry {
    int d, causal, Hq, Hk, bB, bSq, bSk, pack, splits;
};

int bucket(int x) {
    int e = 0;
    while (e < 31 && (1ll << e) < x) ++e;
    return e;
}

// The table shipped beside the library (tune_b200.txt in the directory of this shared
// object), measured on B200 for the benchmark workloads.
std::string default_table_path() {
    Dl_info info{};
    if (dladdr(reinterpret_cast<void*>(&gqa_attn_choose), &info) == 0 || info.dli_fname == nullptr)
        return std::string();
    const std::string so(info.dli_fname);
    const size_t slash = so.find_last_of('/');
    return (slash == std::string::npos ? std::string(".") : so.substr(0, slash)) + "/tune_b200.txt";
}

const std::vector<TuneEntry>& tune_table() {
    static std::vector<TuneEntry> table;
    static std::once_flag once;
    std::call_once(once, [] {
        // GQA_TUNE_TABLE names the table; set but empty, no table; unset, the shipped one
        const char* env = std::getenv("GQA_TUNE_TABLE");
        const std::string path = env != nullptr ? std::string(env) : default_table_path();
        if (path.empty()) return;
        FILE* f = std::fopen(path.c_str(), "r");
        if (f == nullptr) return;
        char line[512];
        while (std::fgets(line, sizeof line, f) != nullptr) {
            if (line[0] == '#') continue;
            TuneEntry e{};
            if (std::sscanf(line, "%d %d %d %d %d %d %d %d %d", &e.d, &e.causal, &e.Hq, &e.Hk,
                            &e.bB, &e.bSq, &e.bSk, &e.pack, &e.splits) == 9 &&
                (e.pack == 0 || e.pack == 1) && e.splits >= 1 && (e.causal == 0 || e.causal == 1))
                table.push_back(e);
        }
        std::fclose(f);
    });
    return table;
}

// The tuned (pack, splits) for this shape's bucket, if the table has one that is valid
// for the shape (packing needs g <= 128).
bool tuned_choice(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal, int* pack,
                  int* splits) {
    const std::vector<TuneEntry>& t = tune_table();
    const int bB = bucket(B), bSq = bucket(Sq), bSk = bucket(Sk);
    for (auto it = t.rbegin(); it != t.rend(); ++it) {
        if (it->d == d && it->causal == causal && it->Hq == Hq && it->Hk == Hk && it->bB == bB &&
            it->bSq == bSq && it->bSk == bSk) {
            if (it->pack == 1 && Hq / Hk > kBlockM) return false;
            *pack = it->pack;
            *splits = it->splits;
            return true;
        }
    }
    return false;
}

int clamp_splits(int s, int kv_blocks) {
    if (s > kv_blocks) s = kv_blocks;
    if (s > kMaxSplits) s = kMaxSplits;
    return s < 1 ? 1 : s;
}

Plan resolve(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal, int pack, int splits,
             int num_sms, bool varlen = false) {
    // a tuned schedule replaces the heuristic for fully automatic calls (dense KV only)
    if (pack < 0 && splits <= 0 && !varlen) {
        int tp = 0, ts = 0;
        if (tuned_choice(B, Sq, Sk, Hq, Hk, d, causal ? 1 : 0, &tp, &ts)) {
            pack = tp;
            splits = ts;
        }
    }
    if (pack < 0) pack = choose_pack(Sq, Hq, Hk, causal);
    Plan pl = make_plan(B, Sq, Sk, Hq, Hk, pack);
    const int auto_splits = varlen ? choose_splits_varlen(pl, d, num_sms) : choose_splits(pl, d, num_sms);
    pl.splits = clamp_splits(splits <= 0 ? auto_splits : splits, pl.kv_blocks);
    pl.units *= pl.splits;
    return pl;
}

// ---------------------------------------------------------------- tensor maps

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encode_tiled() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    });
    return fn;
}

// Tensor [B, S, H, d] as a 4-D map (d, H, S, B), zero fill out of bounds.  bf16: box
// (64, box_h, box_s, 1), 128-byte swizzle (a box row is 128 bytes).  e4m3 (f8): box
// (d, box_h, box_s, 1), one byte per element, 128-byte swizzle for d = 128 and 64-byte for
// d = 64 (a box row is d bytes).
bool encode_bshd(CUtensorMap* m, const void* ptr, int B, int S, int H, int d, int box_h,
                 int box_s, bool f8 = false) {
    EncodeTiled enc = get_encode_tiled();
    if (!enc) return false;
    const cuuint64_t es = f8 ? 1 : 2;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)S * H * d * es};
    cuuint32_t box[4] = {f8 ? (cuuint32_t)d : 64u, (cuuint32_t)box_h, (cuuint32_t)box_s, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw =
        (f8 && d == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    return enc(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
               const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 output [Bs, S, H, d] (Bs = B, or splits * B for the partials) as a 4-D map
// (d, H, S, Bs) for TMA stores: 128-byte swizzle, box (32, box_h, box_s, 1).
// Output map for the epilogue's TMA stores: fp32 with 32-column boxes, or bf16 with
// 64-column boxes; either way a box row is 128 bytes (the 128-byte swizzle span).
bool encode_out(CUtensorMap* m, const void* ptr, int Bs, int S, int H, int d, int box_h,
                int box_s, bool bf16 = false) {
    EncodeTiled enc = get_encode_tiled();
    if (!enc) return false;
    const cuuint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)Bs};
    cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)S * H * d * es};
    cuuint32_t box[4] = {bf16 ? 64u : 32u, (cuuint32_t)box_h, (cuuint32_t)box_s, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
               const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
    int ok = 0;  // 1: sm_100
};

gqa_status device_info(int* dev_out, DeviceInfo* info) {
    static DeviceInfo cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();  // leave no error pending for the caller's own checks
        return GQA_ERR_CUDA;
    }
    *dev_out = dev;
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && cache[dev].sms > 0) {
        *info = cache[dev];
        return GQA_OK;
    }
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return GQA_ERR_CUDA;
    }
    DeviceInfo di;
    di.sms = sms;
    di.ok = (major == 10 && minor == 0) ? 1 : 0;
    if (dev >= 0 && dev < 64) cache[dev] = di;
    *info = di;
    return GQA_OK;
}

// SM count the plan assumes when no device is given: the current device's when there is
// one (what gqa_attn_fwd will plan with), else a B200's 148.
int planning_sms() {
    int dev = 0;
    DeviceInfo info;
    if (device_info(&dev, &info) == GQA_OK && info.sms > 0) return info.sms;
    return kDefaultSms;
}

// Batches per scheduling window: as many as keep the window's K and V within ~12 MB.
// The L2 also carries the Q tiles and the output lines streaming through it (at B=64,
// S=2048 a window of 48 MB of K/V sees about 250 MB of those go by), and K/V lines evicted
// between their readers come back from DRAM: measured on B200 at that shape (causal,
// fp32 output), a 12 MB window reads 2.65 GB from DRAM against 3.5-3.7 GB with 48 MB
// (1.61 GB algorithmic) and runs 0-6 % faster over the prefill sweep.
int batch_window(int B, int Sk, int Hk, int d) {
    const double kv_per_batch = 4.0 * Sk * Hk * d;  // K and V, bf16
    int w = (int)(12.0e6 / (kv_per_batch > 1.0 ? kv_per_batch : 1.0));
    if (w < 1) w = 1;
    return w < B ? w : B;
}

void set_unit_divisors(gqa::FwdParams* p, int B) {
    const int per_batch = p->n_hg * p->n_mt * p->num_splits;
    p->div_window = gqa::make_fastdiv((uint32_t)(p->batch_window * per_batch));
    p->div_splits = gqa::make_fastdiv((uint32_t)p->num_splits);
    p->div_hg = gqa::make_fastdiv((uint32_t)p->n_hg);
    p->div_bw = gqa::make_fastdiv((uint32_t)p->batch_window);
    const int last = B % p->batch_window;
    p->div_bw_last = gqa::make_fastdiv((uint32_t)(last == 0 ? p->batch_window : last));
}

// Split-KV scratch comes from a library-owned stream-ordered pool per device that keeps
// its memory (release threshold = max), so a host synchronisation does not hand the
// memory back to the driver and make the next call map it again.
cudaMemPool_t workspace_pool(int dev) {
    static cudaMemPool_t pools[64] = {};
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (pools[dev] == nullptr) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = ~0ull;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = pool;
    }
    return pools[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Limit of each in-kernel wait: GQA_WAIT_TIMEOUT_NS (nanoseconds) if set, else
// GQA_WAIT_TIMEOUT_MS (milliseconds), else 4 s.  Read at every call.
long long timeout_ns() {
    if (const char* e = std::getenv("GQA_WAIT_TIMEOUT_NS")) {
        const long long ns = std::atoll(e);
        return ns < 1 ? 1 : ns;
    }
    const char* e = std::getenv("GQA_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 4000;
    if (ms < 1) ms = 1;
    return ms * 1000000ll;
}

// Limit of the teardown waits after an abort (copies and MMAs already issued must land
// before shared and tensor memory are released): never below 1 s, whatever the wait
// limit, since those operations complete in microseconds unless the device is stuck.
long long drain_ns(long long wait_ns) { return wait_ns > 1000000000ll ? wait_ns : 1000000000ll; }

// Where the split-KV partials live: the library's stream-ordered pool (scratch ==
// nullptr), or a fixed caller-side buffer of scratch_bytes that is never allocated or
// freed here (the allocation-free entry point).
struct Scratch {
    void* ptr = nullptr;
    size_t bytes = 0;
};

size_t partial_bytes(int splits, int B, int Sq, int Hq, int d) {
    if (splits <= 1) return 0;
    return (size_t)splits * (size_t)B * Hq * Sq * ((size_t)d + 1) * sizeof(float);
}

// e4m3 inputs: q, k, v hold one byte per element; the values are q8 * q_scale etc.
struct Fp8 {
    float q_scale = 1.f, k_scale = 1.f, v_scale = 1.f;
};

// A paged KV cache: k and v are page pools [num_pages, page_size, Hk, d]; key j of
// sequence b is row j % page_size of page block_table[b * table_stride + j / page_size].
struct Paged {
    const int* block_table = nullptr;
    int table_stride = 0;
    int page_size = 0;
    int num_pages = 0;
};

bool is_pow2(long long x) { return x > 0 && (x & (x - 1)) == 0; }

// The forward behind every entry point.  out is fp32 or, with out_bf16, bf16; seqlens_k
// (device, nullable) gives each sequence's key count; fixed (nullable) replaces the pool
// allocation of the split partials; paged (nullable) makes k and v page pools.
gqa_status fwd_impl(const void* q, const void* k, const void* v, const int* seqlens_k, void* out,
                    bool out_bf16, float* lse, int B, int Sq, int Sk, int Hq, int Hk, int d,
                    float scale, int causal, int pack_gqa, int num_splits, void* stream_ptr,
                    const Scratch* fixed = nullptr, const Paged* paged = nullptr,
                    const Fp8* f8 = nullptr) {
    if (!q || !k || !v || !out || !lse) return GQA_ERR_NULL;
    // a paged cache's logical capacity is not a dense tensor: its pool is checked below
    gqa_status st = validate_shape(B, Sq, paged ? 1 : Sk, Hq, Hk, d, pack_gqa, num_splits);
    if (st != GQA_OK) return st;
    if (paged != nullptr) {
        if (f8 != nullptr) return GQA_ERR_SHAPE;  // no e4m3 page pools
        if (!paged->block_table || !seqlens_k) return GQA_ERR_NULL;
        if (!is_pow2(paged->page_size) || paged->page_size < 16 || paged->num_pages < 1 ||
            paged->table_stride < 1 ||
            (long long)paged->num_pages * paged->page_size * Hk >= (1ll << 31))
            return GQA_ERR_SHAPE;
        if ((reinterpret_cast<uintptr_t>(paged->block_table) & 3u) != 0) return GQA_ERR_ALIGN;
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
        return GQA_ERR_ALIGN;
    if (seqlens_k && (reinterpret_cast<uintptr_t>(seqlens_k) & 3u) != 0) return GQA_ERR_ALIGN;
    if (!std::isfinite(scale)) return GQA_ERR_SHAPE;
    int dev = 0;
    DeviceInfo info;
    st = device_info(&dev, &info);
    if (st != GQA_OK) return st;
    if (!info.ok) return GQA_ERR_ARCH;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

    Plan pl = resolve(B, Sq, Sk, Hq, Hk, d, causal ? 1 : 0, pack_gqa, num_splits, info.sms,
                      seqlens_k != nullptr);
    if (fixed != nullptr) {
        // fixed scratch: an automatic split count shrinks until its partials fit (down to
        // no split, which needs none); an explicit one that does not fit is refused
        const size_t cap = fixed->ptr ? fixed->bytes : 0;
        if (num_splits <= 0) {
            const int s0 = pl.splits;
            while (pl.splits > 1 && partial_bytes(pl.splits, B, Sq, Hq, d) > cap) --pl.splits;
            pl.units = pl.units / s0 * pl.splits;
        } else if (partial_bytes(pl.splits, B, Sq, Hq, d) > cap) {
            return GQA_ERR_SCRATCH;
        }
    }
    const int g = Hq / Hk;

    gqa::FwdParams p{};
    const bool is_f8 = f8 != nullptr;
    if (!encode_bshd(&p.tm_q, q, B, Sq, Hq, d, pl.pack ? g : 1, pl.pack ? pl.pos_per_tile : kBlockM, is_f8))
        return GQA_ERR_CUDA;
    if (paged == nullptr) {
        if (!encode_bshd(&p.tm_k, k, B, Sk, Hk, d, 1, kBlockN, is_f8) ||
            !encode_bshd(&p.tm_v, v, B, Sk, Hk, d, 1, kBlockN, is_f8))
            return GQA_ERR_CUDA;
    } else {
        // the page pools as (d, Hk, page_size, num_pages), boxes of up to 128 rows
        const int rows = paged->page_size < kBlockN ? paged->page_size : kBlockN;
        if (!encode_bshd(&p.tm_k, k, paged->num_pages, paged->page_size, Hk, d, 1, rows, is_f8) ||
            !encode_bshd(&p.tm_v, v, paged->num_pages, paged->page_size, Hk, d, 1, rows, is_f8))
            return GQA_ERR_CUDA;
        p.block_table = paged->block_table;
        p.table_stride = paged->table_stride;
        int shift = 0;
        while ((1 << shift) < paged->page_size) ++shift;
        p.page_shift = shift;
        p.page_rows = rows;
        p.num_pages = paged->num_pages;
    }
    p.out = out_bf16 ? nullptr : static_cast<float*>(out);
    p.out_bf16 = out_bf16 ? static_cast<uint16_t*>(out) : nullptr;
    p.seqlens_k = seqlens_k;
    p.lse = lse;
    p.B = B;
    p.Sq = Sq;
    p.Sk = Sk;
    p.Hq = Hq;
    p.Hk = Hk;
    p.g = g;
    p.pack = pl.pack;
    p.pos_per_tile = pl.pos_per_tile;
    p.rows_valid = pl.rows_valid;
    p.causal = causal ? 1 : 0;
    p.num_splits = pl.splits;
    p.n_hg = pl.n_hg;
    p.n_mt = pl.n_mt;
    p.n_units = (int)pl.units;
    p.batch_window = batch_window(B, Sk, Hk, d);
    set_unit_divisors(&p, B);
    p.kv_blocks = pl.kv_blocks;
    // e4m3: the scores are q8 . k8 * q_scale * k_scale, and O carries v_scale
    const double qk = is_f8 ? (double)f8->q_scale * (double)f8->k_scale : 1.0;
    p.scale_log2 = (float)((double)scale * qk * 1.4426950408889634);
    p.v_scale = is_f8 ? f8->v_scale : 1.f;
    // readers of each K/V block: the query-tile units of a (batch, head-or-group), times the
    // heads of a group when they are not packed together
    p.kv_shared = ((long long)pl.n_mt * (pl.pack ? 1 : g) > 1) ? 1 : 0;
    p.div_g = gqa::make_fastdiv((uint32_t)g);
    p.status = nullptr;
    p.timeout_ns = timeout_ns();
    p.drain_ns = drain_ns(p.timeout_ns);
    // host-side fault injection: the kernel stalls on a wait that nothing completes and
    // reports GQA_ERR_TIMEOUT through the status word (tests of the bounded waits)
    p.inject_stall = std::getenv("GQA_FAULT_INJECT_STALL") != nullptr ? 1 : 0;

    // Device scratch: the split partials (num_splits > 1), and with per-sequence lengths the
    // work order of the units (2 ints per unit), in one stream-ordered pool allocation, or
    // the caller's fixed scratch (which never comes with lengths).
    void* ws = nullptr;  // pool allocation to release after the combine (never with fixed)
    const size_t rows = (size_t)B * Hq * Sq;
    const size_t part_bytes = pl.splits > 1 ? (partial_bytes(pl.splits, B, Sq, Hq, d) + 255) & ~(size_t)255 : 0;
    // (the one-tile kernel only: its units share no K/V, while the prefill kernel's unit
    // order keeps a batch window's K/V in L2)
    const size_t order_bytes =
        (seqlens_k != nullptr && pl.nt == 1) ? 2 * (size_t)pl.units * sizeof(int) : 0;
    if (part_bytes + order_bytes > 0) {
        void* base = nullptr;
        if (fixed != nullptr) {
            base = fixed->ptr;
        } else {
            // host-side fault injection: the allocation fails as it would when the device
            // is out of memory (nothing is launched)
            if (std::getenv("GQA_FAULT_INJECT_ALLOC") != nullptr) return GQA_ERR_ALLOC;
            cudaMemPool_t pool = workspace_pool(dev);
            if (pool == nullptr ||
                cudaMallocFromPoolAsync(&ws, part_bytes + order_bytes, pool, stream) != cudaSuccess) {
                cudaGetLastError();
                return GQA_ERR_ALLOC;
            }
            base = ws;
        }
        if (pl.splits > 1) {
            p.o_part = static_cast<float*>(base);
            p.lse_part = p.o_part + (size_t)pl.splits * rows * d;
        }
        if (order_bytes > 0) p.unit_order = reinterpret_cast<int*>(static_cast<char*>(base) + part_bytes);
    }
    if (!encode_out(&p.tm_o, pl.splits > 1 ? (const void*)p.o_part : (const void*)out,
                    pl.splits > 1 ? pl.splits * B : B, Sq, Hq, d, pl.pack ? g : 1,
                    pl.pack ? pl.pos_per_tile : kBlockM, pl.splits == 1 && out_bf16)) {
        if (ws) cudaFreeAsync(ws, stream);
        return GQA_ERR_CUDA;
    }

    const int slots = info.sms * gqa::fwd_ctas_per_sm(d, pl.nt);
    const int grid = (int)(pl.units < slots ? pl.units : slots);
    if (p.unit_order != nullptr) {
        int* order = const_cast<int*>(p.unit_order);
        gqa::FwdParams q = p;
        q.unit_order = nullptr;
        if (gqa::launch_unit_order(q, pl.nt, grid, order, order + pl.units, stream) != cudaSuccess) {
            if (ws) cudaFreeAsync(ws, stream);
            return GQA_ERR_CUDA;
        }
    }
    if (gqa::launch_fwd(p, d, pl.nt, is_f8, grid, stream) != cudaSuccess) {
        if (ws) cudaFreeAsync(ws, stream);
        return GQA_ERR_CUDA;
    }
    if (pl.splits > 1) {
        gqa::CombineParams c{};
        c.o_part = p.o_part;
        c.lse_part = p.lse_part;
        c.out = p.out;
        c.out_bf16 = p.out_bf16;
        c.lse = lse;
        c.B = B;
        c.Sq = Sq;
        c.Hq = Hq;
        c.num_splits = pl.splits;
        cudaError_t e = gqa::launch_combine(c, d, info.sms, stream);
        if (ws) cudaFreeAsync(ws, stream);
        if (e != cudaSuccess) return GQA_ERR_CUDA;
    }
    return GQA_OK;
}

}  // namespace

extern "C" {

const char* gqa_attn_status_string(gqa_status s) {
    switch (s) {
        case GQA_OK: return "ok";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_SHAPE: return "invalid shape, pack_gqa or num_splits";
        case GQA_ERR_HEADS: return "Hq is not a multiple of Hk";
        case GQA_ERR_HEADDIM: return "head dim must be 64 or 128";
        case GQA_ERR_ALIGN: return "pointers must be 16-byte aligned";
        case GQA_ERR_ARCH: return "device is not sm_100 (B200 class)";
        case GQA_ERR_ALLOC: return "split-KV workspace allocation failed";
        case GQA_ERR_CUDA: return "CUDA call failed";
        case GQA_ERR_TIMEOUT: return "an in-kernel bounded wait timed out";
        case GQA_ERR_SCRATCH: return "split-KV partials exceed the library's static scratch";
    }
    return "unknown status";
}

gqa_status gqa_attn_choose(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal, int num_sms,
                           int* pack_gqa, int* num_splits) {
    if (!pack_gqa || !num_splits) return GQA_ERR_NULL;
    gqa_status st = validate_shape(B, Sq, Sk, Hq, Hk, d, -1, 0);
    if (st != GQA_OK) return st;
    Plan pl = resolve(B, Sq, Sk, Hq, Hk, d, causal, -1, 0, num_sms > 0 ? num_sms : planning_sms());
    *pack_gqa = pl.pack;
    *num_splits = pl.splits;
    return GQA_OK;
}

size_t gqa_attn_workspace_bytes(int B, int Sq, int Sk, int Hq, int Hk, int d, int causal,
                                int pack_gqa, int num_splits) {
    if (validate_shape(B, Sq, Sk, Hq, Hk, d, pack_gqa, num_splits) != GQA_OK) return 0;
    Plan pl = resolve(B, Sq, Sk, Hq, Hk, d, causal, pack_gqa, num_splits, planning_sms());
    return partial_bytes(pl.splits, B, Sq, Hq, d);
}

gqa_status gqa_attn_fwd(const void* q, const void* k, const void* v, float* out, float* lse,
                        int B, int Sq, int Sk, int Hq, int Hk, int d, float scale, int causal,
                        int pack_gqa, int num_splits, void* stream) {
    return fwd_impl(q, k, v, nullptr, out, false, lse, B, Sq, Sk, Hq, Hk, d, scale, causal,
                    pack_gqa, num_splits, stream);
}

gqa_status gqa_attn_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache,
                                const int* cache_seqlens, void* out, int out_dtype, float* lse,
                                int B, int Sq, int Sk, int Hq, int Hk, int d, float scale,
                                int causal, int pack_gqa, int num_splits, void* stream) {
    if (out_dtype != GQA_OUT_F32 && out_dtype != GQA_OUT_BF16) return GQA_ERR_SHAPE;
    return fwd_impl(q, k_cache, v_cache, cache_seqlens, out, out_dtype == GQA_OUT_BF16, lse, B,
                    Sq, Sk, Hq, Hk, d, scale, causal, pack_gqa, num_splits, stream);
}

gqa_status gqa_attn_fwd_paged(const void* q, const void* k_pages, const void* v_pages,
                              const int* block_table, int max_pages_per_seq,
                              const int* cache_seqlens, int num_pages, int page_size, void* out,
                              int out_dtype, float* lse, int B, int Sq, int Hq, int Hk, int d,
                              float scale, int causal, int pack_gqa, int num_splits, void* stream) {
    if (out_dtype != GQA_OUT_F32 && out_dtype != GQA_OUT_BF16) return GQA_ERR_SHAPE;
    if (max_pages_per_seq < 1 || page_size < 1 ||
        (long long)max_pages_per_seq * page_size >= (1ll << 31))
        return GQA_ERR_SHAPE;
    Paged pg;
    pg.block_table = block_table;
    pg.table_stride = max_pages_per_seq;
    pg.page_size = page_size;
    pg.num_pages = num_pages;
    return fwd_impl(q, k_pages, v_pages, cache_seqlens, out, out_dtype == GQA_OUT_BF16, lse, B,
                    Sq, max_pages_per_seq * page_size, Hq, Hk, d, scale, causal, pack_gqa,
                    num_splits, stream, nullptr, &pg);
}

gqa_status gqa_attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale,
                            float k_scale, float v_scale, const int* cache_seqlens, void* out,
                            int out_dtype, float* lse, int B, int Sq, int Sk, int Hq, int Hk,
                            int d, float scale, int causal, int pack_gqa, int num_splits,
                            void* stream) {
    if (out_dtype != GQA_OUT_F32 && out_dtype != GQA_OUT_BF16) return GQA_ERR_SHAPE;
    if (!std::isfinite(q_scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale) ||
        !(q_scale > 0.f) || !(k_scale > 0.f) || !(v_scale > 0.f))
        return GQA_ERR_SHAPE;
    Fp8 f8;
    f8.q_scale = q_scale;
    f8.k_scale = k_scale;
    f8.v_scale = v_scale;
    return fwd_impl(q, k, v, cache_seqlens, out, out_dtype == GQA_OUT_BF16, lse, B, Sq, Sk, Hq, Hk,
                    d, scale, causal, pack_gqa, num_splits, stream, nullptr, nullptr, &f8);
}

gqa_status gqa_attn_device_status(int reset) {
    unsigned int* ptr = gqa::device_status_symbol();
    if (!ptr) return GQA_ERR_CUDA;
    unsigned int h = 0;
    if (cudaMemcpy(&h, ptr, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return GQA_ERR_CUDA;
    if (reset) {
        unsigned int z = 0;
        if (cudaMemcpy(ptr, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess)
            return GQA_ERR_CUDA;
    }
    return h ? GQA_ERR_TIMEOUT : GQA_OK;
}

}  // extern "C"

namespace gqa {

gqa_status fwd_fixed_scratch(const void* q, const void* k, const void* v, float* out, float* lse,
                             int B, int Sq, int Sk, int Hq, int Hk, int d, float scale, int causal,
                             int pack_gqa, int num_splits, void* stream, void* scratch,
                             size_t scratch_bytes) {
    Scratch fixed;
    fixed.ptr = scratch;
    fixed.bytes = scratch_bytes;
    return fwd_impl(q, k, v, nullptr, out, false, lse, B, Sq, Sk, Hq, Hk, d, scale, causal,
                    pack_gqa, num_splits, stream, &fixed);
}

}  // namespace gqa
