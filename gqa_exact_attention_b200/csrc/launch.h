// Host-side entry points of the kernels (internal to libgqa_attn.so).
#pragma once

#include <cuda_runtime.h>

#include "fwd_params.h"
#include "gqa_attn.h"

namespace gqa {

// CTAs of the forward kernel resident per SM for (head dim, tiles per CTA).
int fwd_ctas_per_sm(int hd, int nt);
// f8: e4m3 Q, K, V (kind::f8f6f4 MMAs); else bf16.
cudaError_t launch_fwd(const FwdParams& p, int hd, int nt, bool f8, int grid, cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, int hd, int num_sms, cudaStream_t stream);
// Work order for the forward kernel launched with `grid` CTAs (p.unit_order is ignored):
// order[u] for every u < p.n_units, heaviest units first, dealt over the CTAs; tmp holds
// p.n_units ints.
cudaError_t launch_unit_order(const FwdParams& p, int nt, int grid, int* order, int* tmp,
                              cudaStream_t stream);
// Device address of the library's status word on the current device (NULL on error).
unsigned int* device_status_symbol();
// The forward with its split-KV partials in caller-side fixed scratch of scratch_bytes
// (never allocates): an automatic split count shrinks to fit, an explicit one that does
// not fit returns GQA_ERR_SCRATCH (api.cpp).
gqa_status fwd_fixed_scratch(const void* q, const void* k, const void* v, float* out, float* lse,
                             int B, int Sq, int Sk, int Hq, int Hk, int d, float scale, int causal,
                             int pack_gqa, int num_splits, void* stream, void* scratch,
                             size_t scratch_bytes);

}  // namespace gqa
