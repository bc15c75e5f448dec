// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernels.  Not installed; the public interface is include/ssd.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssd {

// Arguments of one chunked-scan call, already validated by the ABI layer.
struct ScanArgs {
    const void* x;
    const void* B;
    const void* C;
    int64_t row_stride;
    const void* dt_raw;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;
    void* y;
    float* final_state;
    int b, L, H, P, N, G, Q;
    bool bf16;
    void* workspace;
    size_t workspace_bytes;
    int32_t* status;
    // Ragged batches: sequence s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1
    // of one packed token dimension of L tokens (b = 1 then); nseq sequences.
    const int* cu_seqlens = nullptr;
    int nseq = 0;
};

// Workspace of a ragged scan: a header (hdr[0] = invalid cu_seqlens flag,
// hdr[1] = unit count) and the per-sequence unit prefix, then the path's own
// workspace.
inline size_t varlen_table_bytes(int nseq) { return ((size_t)256 + (size_t)(nseq + 1) * 4 + 255) / 256 * 256; }
constexpr size_t kVarlenUnitsOffset = 256;   // seq_units after the 256-byte header

cudaError_t launch_varlen_prep(const int* cu_seqlens, int nseq, int T, int H, int Q, int* hdr, int* seq_units,
                               int* ctrl, int ctrl_ints, const float* init_state, float* final_state,
                               long long state_elems_per_seq, int32_t* status, cudaStream_t s);

// Per-unit descriptors of a ragged batch's unit list (the tensor-core scan;
// each CTA writes those of its own range): unit u -> {chain s * H + h,
// chunk c, first token cu[s] + c * Q, end of the sequence cu[s + 1]}.  A
// batch has at most H * (ceil(T / Q) + nseq) units.
inline size_t varlen_desc_bytes(int nseq, long long T, int H, int Q)
{
    const long long units = (long long)H * ((T + Q - 1) / Q + nseq);
    return ((size_t)units * 16 + 255) / 256 * 256;
}

// in_stride: elements between consecutive input tokens (0: conv_dim)
cudaError_t launch_conv1d_silu(const void* xBC, void* out, const float* w, const float* bias,
                               void* conv_state, int b, int L, int conv_dim, int k, bool bf16,
                               cudaStream_t s, int64_t in_stride = 0);

// C0/C1 [M][.] = A[M][K] B[N][K]^T, bf16 in and out, fp32 accumulation
// (tensor cores); output columns >= n_split (a multiple of 8; 0: none) go to
// C1 at column - n_split.
bool gemm_bf16_tn_supported(int M, int N, int K, int64_t lda, int64_t ldb, int n_split);
cudaError_t launch_gemm_bf16_tn(const void* A, int64_t lda, const void* B, int64_t ldb, void* C0, int64_t ldc0,
                                void* C1, int64_t ldc1, int M, int N, int K, int n_split, int32_t* status,
                                cudaStream_t s);

// n[M][d] = RMSNorm over `groups` slices of (y * SiLU(z)) times w, bf16 in/out
cudaError_t launch_rmsnorm_gated(const void* y, int64_t ldy, const void* z, int64_t ldz, const float* w, void* n,
                                 int64_t ldn, int M, int d, int groups, float eps, cudaStream_t s);

bool state_update_supports_n(int N);
cudaError_t launch_state_update(float* state, const void* x, const void* B, const void* C,
                                int64_t row_stride, const void* dt_raw, const float* dt_bias,
                                const float* A, const float* D, void* y, int b, int H, int P,
                                int N, int G, bool bf16, cudaStream_t s);

bool chunk_scan_tc_supported(const ScanArgs& a);
size_t chunk_scan_tc_workspace_bytes(const ScanArgs& a);
cudaError_t launch_chunk_scan_tc(const ScanArgs& a, cudaStream_t s);

size_t chunk_scan_simt_smem_bytes(int P, int N);
cudaError_t launch_chunk_scan_simt(const ScanArgs& a, cudaStream_t s);

}  // namespace ssd
