// conv1d_silu.cu -- causal depthwise conv1d + SiLU over the x | B | C
// channels, with the k-column rolling cache (Mamba cache of "Hybrid
// Architectures for Language Models", summary page, appendix C; conv width 4
// and SiLU from the Nemotron feasibility report, section 1.4).
//
// HBM-bound streaming kernel.  Each thread owns 4 adjacent channels (an
// 8-byte bf16 or 16-byte float vector) and walks a tile of 32 tokens (64 for long sequences),
// keeping the k-1 previous inputs in registers; the k-1 halo tokens before
// its tile are re-read (they were just read by the neighbouring tile, so
// they come from L2).  Tokens move in groups of 8 whose loads are all issued
// before any is used.  A warp covers 128 consecutive channels, so every load
// and store instruction is coalesced along channels.  Four channels per
// thread keep the register count low enough for many resident warps (the
// bytes in flight per SM are what saturates HBM).
//
// The cache is read and rewritten by the thread that owns token tile 0 of a
// channel group, so an in-place cache update never races with a reader.
// The input rows may be wider than conv_dim (in_stride elements apart: the
// xBC columns of the in_projection's output); the output is dense.
#include "common.cuh"
#include "kernels.h"

namespace ssd {

constexpr int kConvThreads = 128;
constexpr int kConvTile = 32;   // tokens per thread
constexpr int kConvTileLong = 64;       // ... for long sequences (fewer halo re-reads, fewer CTAs)
constexpr int kConvLongTokens = 4096;   // L from which the long tile is used (shorter: more CTAs pay)
constexpr int kGroup = 8;       // tokens loaded together
constexpr int kCpt = 4;         // channels per thread

// Packed fp32 pairs (sm_100: one instruction does two lanes of fp32 work,
// each rounded as the scalar operation).
__device__ inline float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ inline float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 4 channels of type T as one vector register group.
template <typename T> struct Vec4;

template <> struct Vec4<float> {
    using raw = uint4;
    __device__ static raw load(const float* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
    __device__ static void decode(raw q, float (&v)[4]) {
        v[0] = __uint_as_float(q.x); v[1] = __uint_as_float(q.y);
        v[2] = __uint_as_float(q.z); v[3] = __uint_as_float(q.w);
    }
    __device__ static void store(float* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
    __device__ static float2 act2(float2 v) { return make_float2(silu_f(v.x), silu_f(v.y)); }
};

template <> struct Vec4<__nv_bfloat16> {
    using raw = uint2;
    __device__ static raw load(const __nv_bfloat16* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
    __device__ static void decode(raw q, float (&v)[4]) {
        v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
    }
    __device__ static void store(__nv_bfloat16* p, const float (&v)[4]) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    }
    // SiLU(v) = v/2 + (v/2) tanh(v/2), as in silu_tanh, on a pair
    __device__ static float2 act2(float2 v)
    {
        const float2 hv = mul2(v, make_float2(0.5f, 0.5f));
        float tx, ty;
        asm("tanh.approx.f32 %0, %1;" : "=f"(tx) : "f"(hv.x));
        asm("tanh.approx.f32 %0, %1;" : "=f"(ty) : "f"(hv.y));
        return fma2(hv, make_float2(tx, ty), hv);
    }
};

// One thread's cache block: 4 channels x K columns of type T, contiguous
// (channel-major), moved as K vectors of 4 * sizeof(T) bytes.  Elements are
// addressed with compile-time indices only, so the block stays in registers.
template <typename T, int K>
struct CacheBlock {
    using R = typename Vec4<T>::raw;
    static constexpr int kWordsPerVec = sizeof(R) / 4;
    uint32_t w[K * kWordsPerVec];
    __device__ void load(const T* p) {
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const R q = reinterpret_cast<const R*>(p)[i];
            const uint32_t* qw = reinterpret_cast<const uint32_t*>(&q);
#pragma unroll
            for (int k = 0; k < kWordsPerVec; ++k) w[i * kWordsPerVec + k] = qw[k];
        }
    }
    __device__ void store(T* p) const {
#pragma unroll
        for (int i = 0; i < K; ++i) {
            R q;
            uint32_t* qw = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
            for (int k = 0; k < kWordsPerVec; ++k) qw[k] = w[i * kWordsPerVec + k];
            reinterpret_cast<R*>(p)[i] = q;
        }
    }
    __device__ float get(int c, int j) const { return io<T>::word_get(w, c * K + j); }
    __device__ void set(int c, int j, float v) { io<T>::word_set(w, c * K + j, v); }
};

// Rewrite one thread's cache block after a call of L tokens, S = min(L, K):
// new column j is old column j + S for j < K - S, else token L - K + j.
// S is a template parameter so every register index is static.
template <typename T, int K, int S>
__device__ inline void roll_cache(T* cs, const T* xb, int L, int64_t in_stride)
{
    CacheBlock<T, K> blk;
    if (S < K) blk.load(cs);
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j < K - S) {
#pragma unroll
            for (int c = 0; c < kCpt; ++c) blk.set(c, j, blk.get(c, j + S));
        } else {
            float v[kCpt];
            Vec4<T>::decode(Vec4<T>::load(xb + (int64_t)(L - K + j) * in_stride), v);
#pragma unroll
            for (int c = 0; c < kCpt; ++c) blk.set(c, j, v[c]);
        }
    }
    blk.store(cs);
}

template <typename T, int K, int kTile>
__global__ void __launch_bounds__(kConvThreads)
conv1d_silu_kernel(const T* __restrict__ xBC, T* __restrict__ out,
                   const float* __restrict__ w, const float* __restrict__ bias,
                   T* __restrict__ conv_state, int L, int conv_dim, int64_t in_stride)
{
    using V4 = Vec4<T>;
    const int ngroups = conv_dim / kCpt;
    const int cg = blockIdx.x * kConvThreads + threadIdx.x;
    if (cg >= ngroups) return;
    const int c0 = cg * kCpt;
    const int t0 = blockIdx.y * kTile;
    const int bi = blockIdx.z;
    const T* xb = xBC + (int64_t)bi * L * in_stride + c0;
    T* ob = out + (size_t)bi * L * conv_dim + c0;

    // taps of the thread's 4 channels: 4*K contiguous floats
    float wt[K][kCpt];
    {
        const float4* w4 = reinterpret_cast<const float4*>(w + (size_t)c0 * K);
        float wl[kCpt * K];
#pragma unroll
        for (int i = 0; i < K; ++i) {
            const float4 q = __ldg(w4 + i);
            wl[4 * i] = q.x; wl[4 * i + 1] = q.y; wl[4 * i + 2] = q.z; wl[4 * i + 3] = q.w;
        }
#pragma unroll
        for (int c = 0; c < kCpt; ++c)
#pragma unroll
            for (int j = 0; j < K; ++j) wt[j][c] = wl[c * K + j];
    }
    float bs[kCpt];
#pragma unroll
    for (int c = 0; c < kCpt; ++c) bs[c] = bias ? bias[c0 + c] : 0.0f;

    // hist[j] holds the input at time t0 - (K-1) + j for j < K-1.
    float hist[K][kCpt];
    if (t0 == 0) {
        if (conv_state) {
            // cache layout [b][conv_dim][K]: column j = time j - K
            CacheBlock<T, K> blk;
            blk.load(conv_state + ((size_t)bi * conv_dim + c0) * K);
#pragma unroll
            for (int c = 0; c < kCpt; ++c)
#pragma unroll
                for (int j = 1; j < K; ++j) hist[j - 1][c] = blk.get(c, j);
        } else {
#pragma unroll
            for (int j = 0; j < K - 1; ++j)
#pragma unroll
                for (int c = 0; c < kCpt; ++c) hist[j][c] = 0.0f;
        }
    } else {
#pragma unroll
        for (int j = 0; j < K - 1; ++j) V4::decode(V4::load(xb + (int64_t)(t0 - (K - 1) + j) * in_stride), hist[j]);
    }

    const int t1 = min(L, t0 + kTile);
    for (int tb = t0; tb < t1; tb += kGroup) {
        typename V4::raw raw[kGroup];
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
            if (tb + u < t1) raw[u] = V4::load(xb + (int64_t)(tb + u) * in_stride);
#pragma unroll
        for (int u = 0; u < kGroup; ++u) {
            if (tb + u < t1) {
                V4::decode(raw[u], hist[K - 1]);
                // the 4 channels as two fp32 pairs
                float2 a01 = make_float2(bs[0], bs[1]), a23 = make_float2(bs[2], bs[3]);
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    a01 = fma2(make_float2(wt[j][0], wt[j][1]), make_float2(hist[j][0], hist[j][1]), a01);
                    a23 = fma2(make_float2(wt[j][2], wt[j][3]), make_float2(hist[j][2], hist[j][3]), a23);
                }
                a01 = V4::act2(a01);
                a23 = V4::act2(a23);
                const float o[kCpt] = {a01.x, a01.y, a23.x, a23.y};
                V4::store(ob + (size_t)(tb + u) * conv_dim, o);
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
#pragma unroll
                    for (int c = 0; c < kCpt; ++c) hist[j][c] = hist[j + 1][c];
            }
        }
    }

    if (t0 == 0 && conv_state) {
        // New cache column j = input at time L - K + j of (old cache | xBC).
        // Times < 0 come from the old cache, which this thread alone reads
        // and writes.
        T* cs = conv_state + ((size_t)bi * conv_dim + c0) * K;
        constexpr int S2 = K < 2 ? K : 2, S3 = K < 3 ? K : 3;
        if (L >= K) roll_cache<T, K, K>(cs, xb, L, in_stride);
        else if (L == 1) roll_cache<T, K, 1>(cs, xb, L, in_stride);
        else if (L == 2) roll_cache<T, K, S2>(cs, xb, L, in_stride);
        else roll_cache<T, K, S3>(cs, xb, L, in_stride);
    }
}

template <typename T, int K>
static cudaError_t launch_conv_k(const void* xBC, void* out, const float* w, const float* bias,
                                 void* conv_state, int b, int L, int conv_dim, int64_t in_stride, cudaStream_t s)
{
    const int ngroups = conv_dim / kCpt;
    // Long sequences take 64-token tiles: 4% faster on 1 x 262144 tokens,
    // 3% slower on 8 x 2048 (same-GPU A/B)
    if (L >= kConvLongTokens) {
        dim3 grid((ngroups + kConvThreads - 1) / kConvThreads, (L + kConvTileLong - 1) / kConvTileLong, b);
        conv1d_silu_kernel<T, K, kConvTileLong><<<grid, kConvThreads, 0, s>>>(
            static_cast<const T*>(xBC), static_cast<T*>(out), w, bias, static_cast<T*>(conv_state),
            L, conv_dim, in_stride);
    } else {
        dim3 grid((ngroups + kConvThreads - 1) / kConvThreads, (L + kConvTile - 1) / kConvTile, b);
        conv1d_silu_kernel<T, K, kConvTile><<<grid, kConvThreads, 0, s>>>(
            static_cast<const T*>(xBC), static_cast<T*>(out), w, bias, static_cast<T*>(conv_state),
            L, conv_dim, in_stride);
    }
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_t(const void* xBC, void* out, const float* w, const float* bias,
                                 void* conv_state, int b, int L, int conv_dim, int64_t in_stride, int k,
                                 cudaStream_t s)
{
    switch (k) {
        case 2: return launch_conv_k<T, 2>(xBC, out, w, bias, conv_state, b, L, conv_dim, in_stride, s);
        case 3: return launch_conv_k<T, 3>(xBC, out, w, bias, conv_state, b, L, conv_dim, in_stride, s);
        case 4: return launch_conv_k<T, 4>(xBC, out, w, bias, conv_state, b, L, conv_dim, in_stride, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_conv1d_silu(const void* xBC, void* out, const float* w, const float* bias,
                               void* conv_state, int b, int L, int conv_dim, int k, bool bf16,
                               cudaStream_t s, int64_t in_stride)
{
    if (in_stride <= 0) in_stride = conv_dim;
    return bf16 ? launch_conv_t<__nv_bfloat16>(xBC, out, w, bias, conv_state, b, L, conv_dim, in_stride, k, s)
                : launch_conv_t<float>(xBC, out, w, bias, conv_state, b, L, conv_dim, in_stride, k, s);
}

}  // namespace ssd
