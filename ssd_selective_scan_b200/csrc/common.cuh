// common.cuh -- small device helpers shared by the libssd kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// ---------------------------------------------------------------------------
// Element access for the two I/O types.  Vectors are 16 bytes: 8 bf16 or
// 4 float.
// ---------------------------------------------------------------------------
template <typename T> struct io;

template <> struct io<float> {
    static constexpr int kVec = 4;
    __device__ static inline float to_f(float v) { return v; }
    __device__ static inline float from_f(float v) { return v; }
    __device__ static inline void load_vec(const float* p, float (&v)[4]) {
        float4 q = *reinterpret_cast<const float4*>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
    __device__ static inline void store_vec(float* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
    __device__ static inline void decode(uint4 q, float (&v)[4]) {
        v[0] = __uint_as_float(q.x); v[1] = __uint_as_float(q.y);
        v[2] = __uint_as_float(q.z); v[3] = __uint_as_float(q.w);
    }
    // element e of a packed word array
    __device__ static inline float word_get(const uint32_t* w, int e) { return __uint_as_float(w[e]); }
    __device__ static inline void word_set(uint32_t* w, int e, float v) { w[e] = __float_as_uint(v); }
};

template <> struct io<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ static inline float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ static inline __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
    __device__ static inline void load_vec(const __nv_bfloat16* p, float (&v)[8]) {
        uint4 q = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static inline void decode(uint4 q, float (&v)[8]) {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static inline float word_get(const uint32_t* w, int e) {
        return __uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
    }
    __device__ static inline void word_set(uint32_t* w, int e, float v) {
        const uint32_t b = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
        w[e >> 1] = (e & 1) ? ((w[e >> 1] & 0x0000ffffu) | (b << 16)) : ((w[e >> 1] & 0xffff0000u) | b);
    }
    __device__ static inline void store_vec(__nv_bfloat16* p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T>
__device__ inline float ld_f(const T* p) { return io<T>::to_f(*p); }

// softplus(v) = log(1 + e^v), evaluated without overflow as
// max(v, 0) + log1p(exp(-|v|)).
__device__ inline float softplus_f(float v) {
    return fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
}

// SiLU(v) = v / (1 + e^-v) with the hardware exp and approximate divide
// (a few ulp, well inside the float32 parity bound).  For v -> -inf the
// denominator overflows to inf and the result is -0.
__device__ inline float silu_f(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// SiLU(v) = v * sigmoid(v) = v * (1/2 + tanh(v/2)/2) with the one-instruction
// hardware tanh (one special-function op instead of an exponential and a
// reciprocal).  tanh.approx is good to about 2^-11 of |tanh| <= 1, so the
// absolute error is about |v| 2^-12: under one bf16 ulp of the result for
// v >= -1, and for very negative v (true result near 0) a few times 10^-3
// at most for |v| <= 10.  Used only where the result is rounded to bf16;
// float32 outputs use silu_f.
__device__ inline float silu_tanh(float v)
{
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
    const float hv = 0.5f * v;
    return fmaf(hv, t, hv);
}

}  // namespace ssd
