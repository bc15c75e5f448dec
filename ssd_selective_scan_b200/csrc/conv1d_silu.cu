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
constexpr int kGroup = 8;       // tokens loaded together

// The V channels x K columns of one thread's cache block are contiguous and
// 16*K bytes long (V * sizeof(T) = 16), so they move as K 16-byte vectors.
// Elements are addressed with compile-time indices only (unrolled loops), so
// the block stays in registers.
template <typename T, int K>
struct CacheBlock {
    static constexpr int kWords = 4 * K;
    uint32_t w[kWords];
    __device__ void load(const T* p) {
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const uint4 q = reinterpret_cast<const uint4*>(p)[i];
            w[4 * i] = q.x; w[4 * i + 1] = q.y; w[4 * i + 2] = q.z; w[4 * i + 3] = q.w;
        }
    }
    __device__ void store(T* p) const {
#pragma unroll
        for (int i = 0; i < K; ++i)
            reinterpret_cast<uint4*>(p)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
    __device__ float get(int c, int j) const { return io<T>::word_get(w, c * K + j); }
    __device__ void set(int c, int j, float v) { io<T>::word_set(w, c * K + j, v); }
};

// Rewrite one thread's cache block after a call of L tokens, S = min(L, K):
// new column j is old column j + S for j < K - S, else token L - K + j.
// S is a template parameter so every register index is static.
template <typename T, int K, int S>
__device__ inline void roll_cache(T* cs, const T* xb, int L, int conv_dim)
{
    constexpr int V = io<T>::kVec;
    CacheBlock<T, K> blk;
    if (S < K) blk.load(cs);
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j < K - S) {
#pragma unroll
            for (int c = 0; c < V; ++c) blk.set(c, j, blk.get(c, j + S));
        } else {
            float v[V];
            io<T>::load_vec(xb + (size_t)(L - K + j) * conv_dim, v);
#pragma unroll
            for (int c = 0; c < V; ++c) blk.set(c, j, v[c]);
        }
    }
    blk.store(cs);
}

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
    {
        // the thread's V channels x K taps are V*K contiguous floats
        const float4* w4 = reinterpret_cast<const float4*>(w + (size_t)c0 * K);
        float wl[V * K];
#pragma unroll
        for (int i = 0; i < V * K / 4; ++i) {
            const float4 q = __ldg(w4 + i);
            wl[4 * i] = q.x; wl[4 * i + 1] = q.y; wl[4 * i + 2] = q.z; wl[4 * i + 3] = q.w;
        }
#pragma unroll
        for (int c = 0; c < V; ++c)
#pragma unroll
            for (int j = 0; j < K; ++j) wt[j][c] = wl[c * K + j];
    }
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

    // Tokens move in groups of kGroup: all loads of a group are issued before
    // any is used, so each thread keeps kGroup x 16 bytes in flight.
    const int t1 = min(L, t0 + kConvTile);
    for (int tb = t0; tb < t1; tb += kGroup) {
        uint4 raw[kGroup];
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
            if (tb + u < t1) raw[u] = __ldcs(reinterpret_cast<const uint4*>(xb + (size_t)(tb + u) * conv_dim));
#pragma unroll
        for (int u = 0; u < kGroup; ++u) {
            if (tb + u < t1) {
                io<T>::decode(raw[u], hist[K - 1]);
                float o[V];
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    float acc = bs[c];
#pragma unroll
                    for (int j = 0; j < K; ++j) acc = fmaf(wt[j][c], hist[j][c], acc);
                    o[c] = silu_f(acc);
                }
                io<T>::store_vec(ob + (size_t)(tb + u) * conv_dim, o);
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
#pragma unroll
                    for (int c = 0; c < V; ++c) hist[j][c] = hist[j + 1][c];
            }
        }
    }

    if (t0 == 0 && conv_state) {
        // New cache column j = input at time L - K + j of (old cache | xBC).
        // Times < 0 come from the old cache, which this thread alone reads
        // and writes.
        T* cs = conv_state + ((size_t)bi * conv_dim + c0) * K;
        constexpr int S2 = K < 2 ? K : 2, S3 = K < 3 ? K : 3;
        if (L >= K) roll_cache<T, K, K>(cs, xb, L, conv_dim);
        else if (L == 1) roll_cache<T, K, 1>(cs, xb, L, conv_dim);
        else if (L == 2) roll_cache<T, K, S2>(cs, xb, L, conv_dim);
        else roll_cache<T, K, S3>(cs, xb, L, conv_dim);
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
