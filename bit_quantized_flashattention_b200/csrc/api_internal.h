// Host-side helpers shared by the C-ABI source files (not exported).
#pragma once

#include <cuda_runtime.h>

#include "../../include/hifa4.h"

namespace hifa4 {

// HIFA4_OK for cudaSuccess; otherwise records `e` as the calling thread's last
// CUDA error (what hifa4_last_cuda_error reports) and returns HIFA4_ERR_CUDA.
hifa4_status from_cuda(cudaError_t e);

// The host-side checks of hifa4_attention_fwd's arguments other than the
// workspace: pointers, alignment, shape, flags, modes and dtypes. Launches
// nothing and touches no device memory.
hifa4_status check_attention_args(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                  float sm_scale, unsigned flags, hifa4_norm_mode norm, const void* o,
                                  hifa4_dtype o_dtype, const float* lse);

}  // namespace hifa4
