// conv1d_silu.cu -- causal depthwise conv1d + SiLU over the x | B | C
// channels, with the k-column rolling cache (Mamba cache of "Hybrid
// Architectures for Language Models", summary page, appendix C; conv width 4
// and SiLU from the Nemotron feasibility report, section 1.4).
//
// HBM-bound streaming kernel.  Each thread owns one 16-byte vector of
// channels (8 bf16 or 4 float) and walks a tile of TT tokens, keeping the
// k-1 previous inputs in registers; the k-1 halo tokens before its tile are
// re-read (they were just read by the neighbouring tile, so they come from
// L2).  Loads and stores are 128-bit and coalesced along channels.
//
// The cache is read and rewritten by the thread that owns token tile 0 of a
// channel vector, so an in-place cache update never races with a reader.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

constexpr int kConvThreads = 128;
constexpr int kConvTile = 32;   // tokens per thread

// The V channels x K columns of one thread's cache block are contiguous and
// 16*K bytes long (V * sizeof(T) = 16), so they move as K 16-byte vectors.
template <typename T, int K>
struct CacheBlock {
    union {
        uint4 q[K];
        T e[io<T>::kVec * K];
    };
    __device__ void load(const T* p) {
#pragma unroll
        for (int i = 0; i < K; ++i) q[i] = reinterpret_cast<const uint4*>(p)[i];
    }
    __device__ void store(T* p) const {
#pragma unroll
        for (int i = 0; i < K; ++i) reinterpret_cast<uint4*>(p)[i] = q[i];
    }
    __device__ float get(int c, int j) const { return io<T>::to_f(e[c * K + j]); }
    __device__ void set(int c, int j, float v) { e[c * K + j] = io<T>::from_f(v); }
};

template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads)
conv1d_silu_kernel(const T* __restrict__ xBC, T* __restrict__ out,
                   const float* __restrict__ w, const float* __restrict__ bias,
                   T* __restrict__ conv_state, int L, int conv_dim)
{
    constexpr int V = io<T>::kVec;
    const int nvec = conv_dim / V;
    const int cv = blockIdx.x * kConvThreads + threadIdx.x;
    if (cv >= nvec) return;
    const int c0 = cv * V;
    const int t0 = blockIdx.y * kConvTile;
    const int bi = blockIdx.z;
    const T* xb = xBC + (size_t)bi * L * conv_dim + c0;
    T* ob = out + (size_t)bi * L * conv_dim + c0;

    float wt[K][V];
#pragma unroll
    for (int c = 0; c < V; ++c)
#pragma unroll
        for (int j = 0; j < K; ++j) wt[j][c] = w[(c0 + c) * K + j];
    float bs[V];
#pragma unroll
    for (int c = 0; c < V; ++c) bs[c] = bias ? bias[c0 + c] : 0.0f;

    // hist[j] holds the input at time t0 - (K-1) + j for j < K-1.
    float hist[K][V];
    if (t0 == 0) {
        if (conv_state) {
            // cache layout [b][conv_dim][K]: column j = time j - K
            CacheBlock<T, K> blk;
            blk.load(conv_state + ((size_t)bi * conv_dim + c0) * K);
#pragma unroll
            for (int c = 0; c < V; ++c)
#pragma unroll
                for (int j = 1; j < K; ++j) hist[j - 1][c] = blk.get(c, j);
        } else {
#pragma unroll
            for (int j = 0; j < K - 1; ++j)
#pragma unroll
                for (int c = 0; c < V; ++c) hist[j][c] = 0.0f;
        }
    } else {
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
            io<T>::load_vec(xb + (size_t)(t0 - (K - 1) + j) * conv_dim, hist[j]);
    }

    const int t1 = min(L, t0 + kConvTile);
    for (int t = t0; t < t1; ++t) {
        io<T>::load_vec(xb + (size_t)t * conv_dim, hist[K - 1]);
        float o[V];
#pragma unroll
        for (int c = 0; c < V; ++c) {
            float acc = bs[c];
#pragma unroll
            for (int j = 0; j < K; ++j) acc = fmaf(wt[j][c], hist[j][c], acc);
            o[c] = silu_f(acc);
        }
        io<T>::store_vec(ob + (size_t)t * conv_dim, o);
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
#pragma unroll
            for (int c = 0; c < V; ++c) hist[j][c] = hist[j + 1][c];
    }

    if (t0 == 0 && conv_state) {
        // New cache column j = input at time L - K + j of (old cache | xBC).
        // Times < 0 come from the old cache, which this thread alone read.
        T* cs = conv_state + ((size_t)bi * conv_dim + c0) * K;
        CacheBlock<T, K> blk;
        blk.load(cs);
        float nc[K][V];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const int tau = L - K + j;
            if (tau >= 0) {
                io<T>::load_vec(xb + (size_t)tau * conv_dim, nc[j]);
            } else {
#pragma unroll
                for (int c = 0; c < V; ++c) nc[j][c] = blk.get(c, tau + K);
            }
        }
#pragma unroll
        for (int c = 0; c < V; ++c)
#pragma unroll
            for (int j = 0; j < K; ++j) blk.set(c, j, nc[j][c]);
        blk.store(cs);
    }
}

template <typename T, int K>
static cudaError_t launch_conv_k(const void* xBC, void* out, const float* w, const float* bias,
                                 void* conv_state, int b, int L, int conv_dim, cudaStream_t s)
{
    constexpr int V = io<T>::kVec;
    const int nvec = conv_dim / V;
    dim3 grid((nvec + kConvThreads - 1) / kConvThreads, (L + kConvTile - 1) / kConvTile, b);
    conv1d_silu_kernel<T, K><<<grid, kConvThreads, 0, s>>>(
        static_cast<const T*>(xBC), static_cast<T*>(out), w, bias, static_cast<T*>(conv_state),
        L, conv_dim);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_t(const void* xBC, void* out, const float* w, const float* bias,
                                 void* conv_state, int b, int L, int conv_dim, int k, cudaStream_t s)
{
    switch (k) {
        case 2: return launch_conv_k<T, 2>(xBC, out, w, bias, conv_state, b, L, conv_dim, s);
        case 3: return launch_conv_k<T, 3>(xBC, out, w, bias, conv_state, b, L, conv_dim, s);
        case 4: return launch_conv_k<T, 4>(xBC, out, w, bias, conv_state, b, L, conv_dim, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_conv1d_silu(const void* xBC, void* out, const float* w, const float* bias,
                               void* conv_state, int b, int L, int conv_dim, int k, bool bf16,
                               cudaStream_t s)
{
    return bf16 ? launch_conv_t<__nv_bfloat16>(xBC, out, w, bias, conv_state, b, L, conv_dim, k, s)
                : launch_conv_t<float>(xBC, out, w, bias, conv_state, b, L, conv_dim, k, s);
}

}  // namespace ssd
