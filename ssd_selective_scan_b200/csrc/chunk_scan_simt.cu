// chunk_scan_simt.cu -- chunked SSD scan on the CUDA cores, float32
// arithmetic throughout.
//
// This is the general path: float32 I/O (where the 1e-4 relative bound rules
// out bf16/TF32 tensor-core operands), and any P, N the tensor-core kernel
// does not take.  It evaluates the same chunk decomposition as the tensor-core
// kernel -- the state-space duality of "Hybrid Architectures for Language
// Models" (summary page, section 2: the scan recast as matrix products) --
// in 64-token chunks, one CTA per (sequence, head) walking the chunks in
// order with the float32 state resident in shared memory:
//
//   dt_i  = softplus(dt_raw_i + dt_bias),  cum_i = sum_{r<=i} dt_r A
//   M[i][j] = (C_i . B_j) exp(cum_i - cum_j) dt_j           (j <= i)
//   y_i   = sum_j M[i][j] x_j + exp(cum_i) C_i . h_prev + D x_i
//   h     = exp(cum_last) h_prev + sum_j exp(cum_last - cum_j) dt_j x_j B_j^T
//
// The chunk length does not change the result beyond rounding, so the
// requested chunk length only bounds this kernel's internal 64.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

constexpr int kSimtThreads = 256;
constexpr int kSimtChunk = 64;

static inline size_t simt_smem_floats(int P, int N)
{
    const int QS = kSimtChunk;
    return (size_t)QS * (N + 1) * 2 + (size_t)QS * (P + 1) + (size_t)QS * (QS + 1) +
           (size_t)P * (N + 1) + 3 * QS;
}

size_t chunk_scan_simt_smem_bytes(int P, int N) { return simt_smem_floats(P, N) * sizeof(float); }

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
chunk_scan_simt_kernel(const T* __restrict__ x, const T* __restrict__ B, const T* __restrict__ C,
                       int64_t rs, const T* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                       const float* __restrict__ A, const float* __restrict__ D,
                       const float* __restrict__ init_state, T* __restrict__ y,
                       float* __restrict__ final_state, int L, int H, int P, int N, int G,
                       const int* __restrict__ cu_seqlens, const int* __restrict__ ws_hdr)
{
    extern __shared__ float smem[];
    constexpr int QS = kSimtChunk;
    const int ldN = N + 1, ldP = P + 1, ldQ = QS + 1;
    float* sB = smem;                       // [QS][ldN]
    float* sC = sB + QS * ldN;              // [QS][ldN]
    float* sX = sC + QS * ldN;              // [QS][ldP]
    float* sM = sX + QS * ldP;              // [QS][ldQ]
    float* sH = sM + QS * ldQ;              // [P][ldN]
    float* sCum = sH + P * ldN;             // [QS]
    float* sDt = sCum + QS;                 // [QS]
    float* sW = sDt + QS;                   // [QS]

    const int h = blockIdx.x % H;
    const int bi = blockIdx.x / H;   // sequence
    // tokens of the sequence: a dense batch's row bi, or a ragged batch's
    // packed tokens cu_seqlens[bi] .. cu_seqlens[bi+1]-1 (nothing is done
    // when the preparation kernel found cu_seqlens invalid)
    size_t row_base = (size_t)bi * L;
    int Ls = L;
    if (cu_seqlens) {
        if (ws_hdr[0]) return;
        row_base = (size_t)cu_seqlens[bi];
        Ls = cu_seqlens[bi + 1] - cu_seqlens[bi];
    }
    const int g = h / (H / G);
    const int tid = threadIdx.x;
    const float Ah = A[h];
    const float Dh = D ? D[h] : 0.0f;
    const float bias = dt_bias ? dt_bias[h] : 0.0f;
    const size_t sidx = ((size_t)bi * H + h) * (size_t)P * N;

    for (int e = tid; e < P * N; e += kSimtThreads) {
        const int p = e / N, n = e % N;
        sH[p * ldN + n] = init_state ? init_state[sidx + e] : 0.0f;
    }

    for (int t0 = 0; t0 < Ls; t0 += QS) {
        const int Qc = min(QS, Ls - t0);
        const size_t row0 = row_base + t0;
        for (int e = tid; e < Qc * N; e += kSimtThreads) {
            const int i = e / N, n = e % N;
            sB[i * ldN + n] = ld_f(B + (row0 + i) * rs + (size_t)g * N + n);
            sC[i * ldN + n] = ld_f(C + (row0 + i) * rs + (size_t)g * N + n);
        }
        for (int e = tid; e < Qc * P; e += kSimtThreads) {
            const int i = e / P, p = e % P;
            sX[i * ldP + p] = ld_f(x + (row0 + i) * rs + (size_t)h * P + p);
        }
        if (tid < Qc) {
            const float dt = softplus_f(ld_f(dt_raw + (row0 + tid) * H + h) + bias);
            sDt[tid] = dt;
            sCum[tid] = dt * Ah;
        }
        __syncthreads();
        if (tid == 0) {
            float run = 0.0f;
            for (int i = 0; i < Qc; ++i) { run += sCum[i]; sCum[i] = run; }
        }
        __syncthreads();
        const float cum_last = sCum[Qc - 1];
        if (tid < Qc) sW[tid] = expf(cum_last - sCum[tid]) * sDt[tid];
        // M[i][j] = (C_i . B_j) exp(cum_i - cum_j) dt_j for j <= i
        for (int e = tid; e < Qc * Qc; e += kSimtThreads) {
            const int i = e / Qc, j = e % Qc;
            float m = 0.0f;
            if (j <= i) {
                float dot = 0.0f;
                for (int n = 0; n < N; ++n) dot = fmaf(sC[i * ldN + n], sB[j * ldN + n], dot);
                m = dot * expf(sCum[i] - sCum[j]) * sDt[j];
            }
            sM[i * ldQ + j] = m;
        }
        __syncthreads();
        // y_i = M x + exp(cum_i) C_i . h_prev + D x_i   (h_prev not yet updated)
        for (int e = tid; e < Qc * P; e += kSimtThreads) {
            const int i = e / P, p = e % P;
            float acc = 0.0f;
            for (int j = 0; j <= i; ++j) acc = fmaf(sM[i * ldQ + j], sX[j * ldP + p], acc);
            float off = 0.0f;
            for (int n = 0; n < N; ++n) off = fmaf(sC[i * ldN + n], sH[p * ldN + n], off);
            const float v = acc + expf(sCum[i]) * off + Dh * sX[i * ldP + p];
            y[((row0 + i) * H + h) * (size_t)P + p] = io<T>::from_f(v);
        }
        __syncthreads();
        // h = exp(cum_last) h_prev + sum_j w_j x_j B_j^T
        const float decay = expf(cum_last);
        for (int e = tid; e < P * N; e += kSimtThreads) {
            const int p = e / N, n = e % N;
            float s = 0.0f;
            for (int j = 0; j < Qc; ++j) s = fmaf(sW[j] * sX[j * ldP + p], sB[j * ldN + n], s);
            sH[p * ldN + n] = fmaf(decay, sH[p * ldN + n], s);
        }
        __syncthreads();
    }
    if (final_state)
        for (int e = tid; e < P * N; e += kSimtThreads) {
            const int p = e / N, n = e % N;
            final_state[sidx + e] = sH[p * ldN + n];
        }
}

template <typename T>
static cudaError_t launch_simt_t(const ScanArgs& a, cudaStream_t s)
{
    const size_t smem = chunk_scan_simt_smem_bytes(a.P, a.N);
    auto kern = chunk_scan_simt_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const bool ragged = a.cu_seqlens != nullptr;
    const int* hdr = nullptr;
    if (ragged) {   // validate cu_seqlens on the device first
        if (!a.workspace || a.workspace_bytes < varlen_table_bytes(a.nseq)) return cudaErrorInvalidValue;
        int* ws = static_cast<int*>(a.workspace);
        e = launch_varlen_prep(a.cu_seqlens, a.nseq, a.L, a.H, kSimtChunk, ws, nullptr, nullptr, 0, a.init_state,
                               a.final_state, (long long)a.H * a.P * a.N, a.status, s);
        if (e != cudaSuccess) return e;
        hdr = ws;
    }
    const dim3 grid((unsigned)((int64_t)(ragged ? a.nseq : a.b) * a.H));
    kern<<<grid, kSimtThreads, smem, s>>>(
        static_cast<const T*>(a.x), static_cast<const T*>(a.B), static_cast<const T*>(a.C),
        a.row_stride, static_cast<const T*>(a.dt_raw), a.dt_bias, a.A, a.D, a.init_state,
        static_cast<T*>(a.y), a.final_state, a.L, a.H, a.P, a.N, a.G, a.cu_seqlens, hdr);
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan_simt(const ScanArgs& a, cudaStream_t s)
{
    return a.bf16 ? launch_simt_t<__nv_bfloat16>(a, s) : launch_simt_t<float>(a, s);
}

}  // namespace ssd
