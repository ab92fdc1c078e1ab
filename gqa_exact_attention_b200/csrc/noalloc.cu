// gqa_attn_fwd_noalloc: the forward for callers that must not allocate device memory.
//
// gqa_attn_fwd allocates its split-KV partials with cudaMallocAsync.  Some callers
// cannot allow that: serving processes that reserve nearly all device memory at start-up
// and forbid allocation on the hot path, code that must not make a call that can block
// on the device, and hosts embedding the library under another runtime's allocator.
// This entry point keeps the partials in one fixed, file-scope device array instead and
// calls no allocating routine.  Contract and limits: include/gqa_attn.h.
#include <cuda_runtime.h>

#include <mutex>

#include "gqa_attn.h"
#include "launch.h"

namespace {

// The split-KV scratch: GQA_NOALLOC_SCRATCH_BYTES on every GPU that loads the library,
// held until the process exits.  Shared by every call; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GQA_NOALLOC_SCRATCH_BYTES];

// Host code must not pass g_noalloc_scratch itself (a host-side stand-in, not a device
// address): its device address is looked up per device, with that device current.  Only
// a successful look-up is kept, so a call that failed (for instance one made during a
// stream capture) does not break the device for later calls; they retry.
constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

gqa_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return GQA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_addr_mu);
    if (g_addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();  // leave no error pending for the caller's own checks
            return GQA_ERR_CUDA;
        }
        g_addr[dev] = ptr;
    }
    *out = g_addr[dev];
    return GQA_OK;
}

}  // namespace

extern "C" gqa_status gqa_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                           float* out, float* lse, int B, int Sq, int Sk,
                                           int Hq, int Hk, int d, float scale, int causal,
                                           int pack_gqa, int num_splits, void* stream) {
    if (!q || !k || !v || !out || !lse) return GQA_ERR_NULL;
    void* scratch = nullptr;
    gqa_status st = scratch_for_current_device(&scratch);
    if (st != GQA_OK) return st;
    return gqa::fwd_fixed_scratch(q, k, v, out, lse, B, Sq, Sk, Hq, Hk, d, scale, causal,
                                  pack_gqa, num_splits, stream, scratch,
                                  GQA_NOALLOC_SCRATCH_BYTES);
}
