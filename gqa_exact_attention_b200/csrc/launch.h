// Host-side entry points of the kernels (internal to libgqa_attn.so).
#pragma once

#include <cuda_runtime.h>

#include "fwd_params.h"

namespace gqa {

// CTAs of the forward kernel resident per SM for (head dim, tiles per CTA).
int fwd_ctas_per_sm(int hd, int nt);
cudaError_t launch_fwd(const FwdParams& p, int hd, int nt, int grid, cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, int hd, int num_sms, cudaStream_t stream);
// Device address of the library's status word on the current device (NULL on error).
unsigned int* device_status_symbol();

}  // namespace gqa
