// decode.h -- internal launch interface of the one-kernel decode step
// (state_update.cu), used by the C ABI (api.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ssd {

// The decode step in one kernel (conv-cache roll, conv + SiLU, state
// update), one CTA per (sequence, group); conv_state [b][conv_dim][k].
// Shared memory per CTA, bytes.
size_t decode_step_smem_bytes(int H, int P, int N, int G);
cudaError_t launch_decode_step(float* state, void* conv_state, const void* xBC, const float* w,
                               const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                               const float* D, void* y, int b, int H, int P, int N, int G, int k, bool bf16,
                               cudaStream_t s);

// The decode step in one kernel, one CTA per (sequence, head); arrivals:
// int32 [b][G], zero on entry and left zero.
size_t decode_step_head_smem_bytes(int P, int N);
int decode_step_head_max_p();   // largest head dim of the per-head form
cudaError_t launch_decode_step_head(float* state, void* conv_state, const void* xBC, const float* w,
                                    const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                    const float* D, void* y, int* arrivals, int b, int H, int P, int N, int G, int k,
                                    bool bf16, cudaStream_t s);

}  // namespace ssd
