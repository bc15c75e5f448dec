// scan_bwd.h -- internal launch interface of the backward pass of the scan
// (scan_bwd.cu), used by the C ABI (api.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssd {

// Arguments of one backward call, already validated by the ABI layer.
// x, B, C, dt_raw as for the forward scan (token rows row_stride apart);
// dy, dx [b][L][H][P], dB, dC [b][L][G][N], ddt_raw [b][L][H] in the I/O
// type; dA, dD, ddt_bias [H], dfinal, dinit [b][H][P][N] float32.
struct ScanBwdArgs {
    const void* x;
    const void* B;
    const void* C;
    int64_t row_stride;
    const void* dt_raw;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;
    const void* dy;
    const float* dfinal;
    void* dx;
    void* dB;
    void* dC;
    void* ddt_raw;
    float* dA;
    float* dD;
    float* ddt_bias;
    float* dinit;
    int b, L, H, P, N, G;
    bool bf16;
    void* workspace;
};

// General path (scan_bwd.cu): float32 on the CUDA cores, any P and N whose
// shared-memory footprint fits one CTA.
size_t scan_bwd_smem_bytes(int P, int N);
size_t scan_bwd_workspace_bytes(int b, int L, int H, int P, int N);
cudaError_t launch_scan_bwd(const ScanBwdArgs& a, cudaStream_t s);

// Tensor-core path (scan_bwd_tc.cu): bf16 I/O with P = 64, N = 128.
// scan_bwd_tc_shape: the dtype and shape qualify (the workspace is sized for
// both paths then); scan_bwd_tc_supported: the call also meets the TMA and
// vector-store alignment (16-byte pointers, row_stride % 8 == 0) and size
// limits, else the general path runs.
bool scan_bwd_tc_shape(int P, int N, bool bf16);
bool scan_bwd_tc_supported(const ScanBwdArgs& a);
size_t scan_bwd_tc_workspace_bytes(int b, int L, int H);
cudaError_t launch_scan_bwd_tc(const ScanBwdArgs& a, cudaStream_t s);

}  // namespace ssd
