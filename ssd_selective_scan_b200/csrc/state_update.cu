// state_update.cu -- single-token selective state update (decode step).
//
// The recurrence of "Hybrid Architectures for Language Models" (summary page,
// section 2 Background), h = Abar h + Bbar x, y = C h + D x, run once per
// (sequence, head) with Abar = exp(dt*A), Bbar = dt*B and
// dt = softplus(dt_raw + dt_bias).  The state is float32 [b][H][P][N] and is
// rewritten in place; it stays a constant size however long the context is
// (the Mamba cache of the same page's appendix C).
//
// HBM-bound: each state element is read once and written once (8 bytes) for
// ~4 flops.  One CTA per (sequence, head); each warp takes rows p of the
// head's P x N state, with TPR lanes per row each holding N/TPR contiguous
// floats as 128-bit vectors.  All of a thread's rows are loaded before any is
// used, so every thread keeps ROWS x 16 bytes of streaming loads in flight.
// The y reduction over N is a butterfly over the TPR lanes of a row.
#include "common.cuh"
#include "kernels.h"
#include "decode.h"

namespace ssd {

constexpr int kSuThreads = 128;

template <typename T, int N>
__global__ void __launch_bounds__(kSuThreads)
state_update_kernel(float* __restrict__ state, const T* __restrict__ x,
                    const T* __restrict__ B, const T* __restrict__ C, int64_t row_stride,
                    const T* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                    const float* __restrict__ A, const float* __restrict__ D,
                    T* __restrict__ y, int H, int P, int G)
{
    constexpr int NV = N / 4;                      // float4 per state row
    constexpr int TPR = NV < 32 ? NV : 32;         // lanes per row
    constexpr int VPL = NV / TPR;                  // float4 per lane per row
    constexpr int RPW = 32 / TPR;                  // rows per warp pass
    constexpr int ROWS = 8;                        // passes loaded together

    const int h = blockIdx.x % H;
    const int bi = blockIdx.x / H;
    const int g = h / (H / G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / TPR, li = lane % TPR;
    constexpr int kWarps = kSuThreads / 32;

    const float dt = softplus_f(ld_f(dt_raw + (size_t)bi * H + h) + (dt_bias ? dt_bias[h] : 0.0f));
    const float dA = expf(dt * A[h]);
    const float Dh = D ? D[h] : 0.0f;

    const T* xr = x + (size_t)bi * row_stride + (size_t)h * P;
    const T* Br = B + (size_t)bi * row_stride + (size_t)g * N;
    const T* Cr = C + (size_t)bi * row_stride + (size_t)g * N;
    float bv[VPL][4], cvv[VPL][4];
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = (v * TPR + li) * 4 + e;
            bv[v][e] = ld_f(Br + n);
            cvv[v][e] = ld_f(Cr + n);
        }

    float* sh = state + ((size_t)bi * H + h) * (size_t)P * N;
    T* yr = y + ((size_t)bi * H + h) * P;
    const int rows_per_iter = kWarps * RPW * ROWS;
    for (int p0 = 0; p0 < P; p0 += rows_per_iter) {
        float4 st[ROWS][VPL];
        int prow[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            prow[r] = p0 + (r * kWarps + warp) * RPW + sub;
            if (prow[r] < P) {
#pragma unroll
                for (int v = 0; v < VPL; ++v)
                    st[r][v] = __ldcs(reinterpret_cast<const float4*>(sh + (size_t)prow[r] * N) + v * TPR + li);
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const bool ok = prow[r] < P;
            const float xp = ok ? ld_f(xr + prow[r]) : 0.0f;
            const float dtx = dt * xp;
            float acc = 0.0f;
            if (ok) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float4 s = st[r][v];
                    s.x = fmaf(dA, s.x, dtx * bv[v][0]);
                    s.y = fmaf(dA, s.y, dtx * bv[v][1]);
                    s.z = fmaf(dA, s.z, dtx * bv[v][2]);
                    s.w = fmaf(dA, s.w, dtx * bv[v][3]);
                    acc = fmaf(cvv[v][0], s.x, acc);
                    acc = fmaf(cvv[v][1], s.y, acc);
                    acc = fmaf(cvv[v][2], s.z, acc);
                    acc = fmaf(cvv[v][3], s.w, acc);
                    __stcs(reinterpret_cast<float4*>(sh + (size_t)prow[r] * N) + v * TPR + li, s);
                }
            }
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (ok && li == 0) yr[prow[r]] = io<T>::from_f(fmaf(Dh, xp, acc));
        }
    }
}

template <typename T>
static cudaError_t launch_su_t(float* state, const void* x, const void* B, const void* C,
                               int64_t rs, const void* dt_raw, const float* dt_bias, const float* A,
                               const float* D, void* y, int b, int H, int P, int N, int G,
                               cudaStream_t s)
{
    const dim3 grid((unsigned)((int64_t)b * H));
#define SSD_SU_CASE(NN)                                                                        \
    case NN:                                                                                   \
        state_update_kernel<T, NN><<<grid, kSuThreads, 0, s>>>(                                \
            state, static_cast<const T*>(x), static_cast<const T*>(B), static_cast<const T*>(C), \
            rs, static_cast<const T*>(dt_raw), dt_bias, A, D, static_cast<T*>(y), H, P, G);    \
        break;
    switch (N) {
        SSD_SU_CASE(4) SSD_SU_CASE(8) SSD_SU_CASE(16) SSD_SU_CASE(32)
        SSD_SU_CASE(64) SSD_SU_CASE(128) SSD_SU_CASE(256)
        default: return cudaErrorInvalidValue;
    }
#undef SSD_SU_CASE
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The decode step in one kernel: the conv-cache roll, conv (width K) and
// SiLU of the new token, then the state update.  One CTA per (sequence,
// group): it convolves the group's B and C channels once and the x channels
// of the group's H / G heads, rewrites exactly those channels' cache columns
// (so no two CTAs touch the same cache entry and the in-place roll cannot
// race), keeps the conv outputs in shared memory, then streams the heads'
// states.  Every value is computed as by conv1d_silu_kernel (L = 1, with a
// cache) followed by state_update_kernel: the conv outputs are rounded to
// the I/O type, and each state row uses the same lane layout and reduction
// order, so the results are equal bit for bit.
// ---------------------------------------------------------------------------
constexpr int kDecThreads = 256;
constexpr int kDecBlocksPerSm = 3;

template <typename T> __device__ inline float conv_act(float v);
template <> __device__ inline float conv_act<float>(float v) { return silu_f(v); }
template <> __device__ inline float conv_act<__nv_bfloat16>(float v)
{
    // the conv kernel's bf16 form: v/2 + (v/2) tanh(v/2)
    const float hv = v * 0.5f;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hv));
    return fmaf(hv, t, hv);
}

template <typename T, int N, int K>
__global__ void __launch_bounds__(kDecThreads, kDecBlocksPerSm)
decode_step_kernel(float* __restrict__ state, T* __restrict__ conv_state, const T* __restrict__ xBC,
                   const float* __restrict__ w, const float* __restrict__ bias,
                   const T* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                   const float* __restrict__ A, const float* __restrict__ D, T* __restrict__ y,
                   int H, int P, int G)
{
    // shared: x of the group's heads [hpg * P], B [N], C [N], then per head dt, exp(dt A), D
    extern __shared__ float sU[];
    constexpr int NV = N / 4;
    constexpr int TPR = NV < 32 ? NV : 32;
    constexpr int VPL = NV / TPR;
    constexpr int RPW = 32 / TPR;
    constexpr int ROWS = 8 / VPL;   // 128 bytes of state in flight per thread
    constexpr int kWarps = kDecThreads / 32;

    const int g = blockIdx.x % G;
    const int bi = blockIdx.x / G;
    const int hpg = H / G;
    const int conv_dim = H * P + 2 * G * N;
    const int nx = hpg * P;
    float* sDt = sU + nx + 2 * N;
    float* sDA = sDt + hpg;
    float* sD = sDA + hpg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / TPR, li = lane % TPR;
    const int rows_per_iter = kWarps * RPW * ROWS;

    // A thread's rows in one pass are p = p0 + r * kRowStep + prow0,
    // r < ROWS: one base address and compile-time offsets.
    constexpr int kRowStep = kWarps * RPW;
    const int prow0 = warp * RPW + sub;
    // the first rows of the first head's state are requested before the
    // conv, so that their latency overlaps it
    float4 st[ROWS][VPL];
    auto load_rows = [&](const float* sh, int p0) {
        const float4* src = reinterpret_cast<const float4*>(sh + (size_t)(p0 + prow0) * N) + li;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            if (p0 + prow0 + r * kRowStep < P) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) st[r][v] = __ldcs(src + r * kRowStep * NV + v * TPR);
            }
        }
    };
    load_rows(state + ((size_t)bi * H + g * hpg) * (size_t)P * N, 0);

    // 1. conv + SiLU of the group's channels, the cache roll, and each
    //    head's dt terms
    for (int i = threadIdx.x; i < nx + 2 * N; i += kDecThreads) {
        const int c = i < nx ? g * nx + i : (i < nx + N ? H * P + g * N + (i - nx) : H * P + G * N + g * N + (i - nx - N));
        T* cs = conv_state + ((size_t)bi * conv_dim + c) * K;
        float win[K];
#pragma unroll
        for (int j = 0; j + 1 < K; ++j) win[j] = ld_f(cs + j + 1);
        win[K - 1] = ld_f(xBC + (size_t)bi * conv_dim + c);
        float acc = bias ? bias[c] : 0.0f;
#pragma unroll
        for (int j = 0; j < K; ++j) acc = fmaf(w[(size_t)c * K + j], win[j], acc);
        sU[i] = io<T>::to_f(io<T>::from_f(conv_act<T>(acc)));
#pragma unroll
        for (int j = 0; j < K; ++j) cs[j] = io<T>::from_f(win[j]);
    }
    for (int hl = threadIdx.x; hl < hpg; hl += kDecThreads) {
        const int h = g * hpg + hl;
        const float dt = softplus_f(ld_f(dt_raw + (size_t)bi * H + h) + (dt_bias ? dt_bias[h] : 0.0f));
        sDt[hl] = dt;
        sDA[hl] = expf(dt * A[h]);
        sD[hl] = D ? D[h] : 0.0f;
    }
    __syncthreads();

    // 2. the state update of each head of the group
    const float* Bs = sU + nx;
    const float* Cs = sU + nx + N;
    float bv[VPL][4], cvv[VPL][4];
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = (v * TPR + li) * 4 + e;
            bv[v][e] = Bs[n];
            cvv[v][e] = Cs[n];
        }
    for (int hl = 0; hl < hpg; ++hl) {
        const int h = g * hpg + hl;
        const float dt = sDt[hl], dA = sDA[hl], Dh = sD[hl];
        const float* xs = sU + hl * P;
        float* sh = state + ((size_t)bi * H + h) * (size_t)P * N;
        T* yr = y + ((size_t)bi * H + h) * P;
        for (int p0 = 0; p0 < P; p0 += rows_per_iter) {
            if (hl > 0 || p0 > 0) load_rows(sh, p0);
            float4* dst = reinterpret_cast<float4*>(sh + (size_t)(p0 + prow0) * N) + li;
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const int prow = p0 + prow0 + r * kRowStep;
                const bool ok = prow < P;
                const float xp = ok ? xs[prow] : 0.0f;
                const float dtx = dt * xp;
                float acc = 0.0f;
                if (ok) {
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        float4 q = st[r][v];
                        q.x = fmaf(dA, q.x, dtx * bv[v][0]);
                        q.y = fmaf(dA, q.y, dtx * bv[v][1]);
                        q.z = fmaf(dA, q.z, dtx * bv[v][2]);
                        q.w = fmaf(dA, q.w, dtx * bv[v][3]);
                        acc = fmaf(cvv[v][0], q.x, acc);
                        acc = fmaf(cvv[v][1], q.y, acc);
                        acc = fmaf(cvv[v][2], q.z, acc);
                        acc = fmaf(cvv[v][3], q.w, acc);
                        __stcs(dst + r * kRowStep * NV + v * TPR, q);
                    }
                }
#pragma unroll
                for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (ok && li == 0) yr[prow] = io<T>::from_f(fmaf(Dh, xp, acc));
            }
        }
    }
}

size_t decode_step_smem_bytes(int H, int P, int N, int G) { return ((size_t)(H / G) * (P + 3) + 2 * (size_t)N) * 4; }

template <typename T, int K>
static cudaError_t launch_dec_k(float* state, void* conv_state, const void* xBC, const float* w,
                                const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                const float* D, void* y, int b, int H, int P, int N, int G, cudaStream_t s)
{
    const dim3 grid((unsigned)((int64_t)b * G));
    const size_t smem = decode_step_smem_bytes(H, P, N, G);
#define SSD_DEC_CASE(NN)                                                                                   \
    case NN: {                                                                                             \
        auto kern = decode_step_kernel<T, NN, K>;                                                          \
        if (smem > 48 * 1024) {                                                                            \
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                                       (int)smem);                                         \
            if (e != cudaSuccess) return e;                                                                \
        }                                                                                                  \
        kern<<<grid, kDecThreads, smem, s>>>(state, static_cast<T*>(conv_state), static_cast<const T*>(xBC), \
                                            w, bias, static_cast<const T*>(dt_raw), dt_bias, A, D,         \
                                            static_cast<T*>(y), H, P, G);                                  \
        break;                                                                                             \
    }
    switch (N) {
        SSD_DEC_CASE(4) SSD_DEC_CASE(8) SSD_DEC_CASE(16) SSD_DEC_CASE(32)
        SSD_DEC_CASE(64) SSD_DEC_CASE(128) SSD_DEC_CASE(256)
        default: return cudaErrorInvalidValue;
    }
#undef SSD_DEC_CASE
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_dec_t(float* state, void* conv_state, const void* xBC, const float* w,
                                const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                const float* D, void* y, int b, int H, int P, int N, int G, int k, cudaStream_t s)
{
    switch (k) {
        case 2: return launch_dec_k<T, 2>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, s);
        case 3: return launch_dec_k<T, 3>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, s);
        case 4: return launch_dec_k<T, 4>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_step(float* state, void* conv_state, const void* xBC, const float* w,
                               const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                               const float* D, void* y, int b, int H, int P, int N, int G, int k, bool bf16,
                               cudaStream_t s)
{
    return bf16 ? launch_dec_t<__nv_bfloat16>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P,
                                              N, G, k, s)
                : launch_dec_t<float>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, k,
                                      s);
}

// ---------------------------------------------------------------------------
// The decode step in one kernel, one CTA per (sequence, head), with a
// workspace of one int32 counter per (sequence, group).  Every CTA convolves
// its head's x channels and its group's B and C channels (the B and C conv
// is repeated by each of the group's H / G heads, from L2), rolls the cache
// of its own x channels, and streams its head's state like
// state_update_kernel, so that many small CTAs keep HBM busy.  The group's B
// and C cache columns are shared by its heads: each CTA counts itself in
// once it has read them (a fence, then an atomic increment), and the last of
// the group's CTAs to arrive rewrites them and resets the counter to zero.
// No CTA waits for another.  Values are computed as by decode_step_kernel,
// so the results are equal bit for bit.
// ---------------------------------------------------------------------------
constexpr int kDecHeadThreads = 128;
constexpr int kDecHeadMaxP = 256;   // head dim supported by the per-head form

template <typename T, int N, int K>
__global__ void __launch_bounds__(kDecHeadThreads, 6)
decode_step_head_kernel(float* __restrict__ state, T* __restrict__ conv_state, const T* __restrict__ xBC,
                        const float* __restrict__ w, const float* __restrict__ bias,
                        const T* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                        const float* __restrict__ A, const float* __restrict__ D, T* __restrict__ y,
                        int* __restrict__ arrivals, int H, int P, int G)
{
    // shared: x of the head [P], the group's B [N] and C [N]; the last-arrival flag
    extern __shared__ float sU[];
    __shared__ int s_last;
    constexpr int NV = N / 4;
    constexpr int TPR = NV < 32 ? NV : 32;
    constexpr int VPL = NV / TPR;
    constexpr int RPW = 32 / TPR;
    constexpr int ROWS = 8 / VPL;
    constexpr int kWarps = kDecHeadThreads / 32;
    constexpr int kBcPer = (2 * N + kDecHeadThreads - 1) / kDecHeadThreads;   // B/C channels per thread
    constexpr int kXPer = kDecHeadMaxP / kDecHeadThreads;                      // x channels per thread, at most

    const int h = blockIdx.x % H;
    const int bi = blockIdx.x / H;
    const int hpg = H / G;
    const int g = h / hpg;
    const int conv_dim = H * P + 2 * G * N;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = lane / TPR, li = lane % TPR;
    constexpr int kRowStep = kWarps * RPW;
    const int prow0 = warp * RPW + sub;
    float* sh = state + ((size_t)bi * H + h) * (size_t)P * N;

    // the first state rows are requested before the conv
    float4 st[ROWS][VPL];
    auto load_rows = [&](int p0) {
        const float4* src = reinterpret_cast<const float4*>(sh + (size_t)(p0 + prow0) * N) + li;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            if (p0 + prow0 + r * kRowStep < P) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) st[r][v] = __ldcs(src + r * kRowStep * NV + v * TPR);
            }
        }
    };
    load_rows(0);

    // conv + SiLU of one channel from the cache columns 1..K-1 and the new
    // token; the window is kept for the cache roll
    auto conv_channel = [&](int c, float (&win)[K]) {
        const T* cs = conv_state + ((size_t)bi * conv_dim + c) * K;
#pragma unroll
        for (int j = 0; j + 1 < K; ++j) win[j] = ld_f(cs + j + 1);
        win[K - 1] = ld_f(xBC + (size_t)bi * conv_dim + c);
        float acc = bias ? bias[c] : 0.0f;
#pragma unroll
        for (int j = 0; j < K; ++j) acc = fmaf(w[(size_t)c * K + j], win[j], acc);
        return io<T>::to_f(io<T>::from_f(conv_act<T>(acc)));
    };
    auto roll = [&](int c, const float (&win)[K]) {
        T* cs = conv_state + ((size_t)bi * conv_dim + c) * K;
#pragma unroll
        for (int j = 0; j < K; ++j) cs[j] = io<T>::from_f(win[j]);
    };
    auto bc_channel = [&](int i) { return i < N ? H * P + g * N + i : H * P + G * N + g * N + (i - N); };
    // 1. the head's x channels and the group's B and C channels; every
    //    cache read of the CTA comes before its arrival is counted
    float wx[kXPer][K], wbc[kBcPer][K];
#pragma unroll
    for (int q = 0; q < kXPer; ++q) {
        const int i = tid + q * kDecHeadThreads;
        if (i < P) sU[i] = conv_channel(h * P + i, wx[q]);
    }
#pragma unroll
    for (int q = 0; q < kBcPer; ++q) {
        const int i = tid + q * kDecHeadThreads;
        if (i < 2 * N) sU[P + i] = conv_channel(bc_channel(i), wbc[q]);
    }
    const float dt = softplus_f(ld_f(dt_raw + (size_t)bi * H + h) + (dt_bias ? dt_bias[h] : 0.0f));
    const float dA = expf(dt * A[h]);
    const float Dh = D ? D[h] : 0.0f;
    __syncthreads();
    // 2. count this CTA in (acquire-release: its reads of the shared cache
    //    columns are ordered before the increment, and the last CTA's
    //    rewrite of them after its own); then roll the head's x channels,
    //    which this CTA alone owns
    if (tid == 0) {
        int prev;
        asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(prev) : "l"(arrivals + (size_t)bi * G + g)
                     : "memory");
        s_last = prev == hpg - 1;
    }
#pragma unroll
    for (int q = 0; q < kXPer; ++q) {
        const int i = tid + q * kDecHeadThreads;
        if (i < P) roll(h * P + i, wx[q]);
    }

    // 3. the state update of the head
    const float* Bs = sU + P;
    const float* Cs = sU + P + N;
    float bv[VPL][4], cvv[VPL][4];
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = (v * TPR + li) * 4 + e;
            bv[v][e] = Bs[n];
            cvv[v][e] = Cs[n];
        }
    T* yr = y + ((size_t)bi * H + h) * P;
    const int rows_per_iter = kWarps * RPW * ROWS;
    for (int p0 = 0; p0 < P; p0 += rows_per_iter) {
        if (p0 > 0) load_rows(p0);
        float4* dst = reinterpret_cast<float4*>(sh + (size_t)(p0 + prow0) * N) + li;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int prow = p0 + prow0 + r * kRowStep;
            const bool ok = prow < P;
            const float xp = ok ? sU[prow] : 0.0f;
            const float dtx = dt * xp;
            float acc = 0.0f;
            if (ok) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float4 q = st[r][v];
                    q.x = fmaf(dA, q.x, dtx * bv[v][0]);
                    q.y = fmaf(dA, q.y, dtx * bv[v][1]);
                    q.z = fmaf(dA, q.z, dtx * bv[v][2]);
                    q.w = fmaf(dA, q.w, dtx * bv[v][3]);
                    acc = fmaf(cvv[v][0], q.x, acc);
                    acc = fmaf(cvv[v][1], q.y, acc);
                    acc = fmaf(cvv[v][2], q.z, acc);
                    acc = fmaf(cvv[v][3], q.w, acc);
                    __stcs(dst + r * kRowStep * NV + v * TPR, q);
                }
            }
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (ok && li == 0) yr[prow] = io<T>::from_f(fmaf(Dh, xp, acc));
        }
    }

    // 4. the group's last CTA rolls the B and C cache columns and resets the
    //    counter for the next call
    __syncthreads();
    if (s_last) {
#pragma unroll
        for (int q = 0; q < kBcPer; ++q) {
            const int i = tid + q * kDecHeadThreads;
            if (i < 2 * N) roll(bc_channel(i), wbc[q]);
        }
        if (tid == 0) atomicExch(arrivals + (size_t)bi * G + g, 0);
    }
}

size_t decode_step_head_smem_bytes(int P, int N) { return ((size_t)P + 2 * (size_t)N) * 4; }
int decode_step_head_max_p() { return kDecHeadMaxP; }

template <typename T, int K>
static cudaError_t launch_dec_head_k(float* state, void* conv_state, const void* xBC, const float* w,
                                     const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                     const float* D, void* y, int* arrivals, int b, int H, int P, int N, int G,
                                     cudaStream_t s)
{
    const dim3 grid((unsigned)((int64_t)b * H));
    const size_t smem = decode_step_head_smem_bytes(P, N);
#define SSD_DECH_CASE(NN)                                                                                  \
    case NN: {                                                                                             \
        auto kern = decode_step_head_kernel<T, NN, K>;                                                     \
        if (smem > 48 * 1024) {                                                                            \
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                                       (int)smem);                                         \
            if (e != cudaSuccess) return e;                                                                \
        }                                                                                                  \
        kern<<<grid, kDecHeadThreads, smem, s>>>(state, static_cast<T*>(conv_state),                       \
                                                 static_cast<const T*>(xBC), w, bias,                      \
                                                 static_cast<const T*>(dt_raw), dt_bias, A, D,             \
                                                 static_cast<T*>(y), arrivals, H, P, G);                   \
        break;                                                                                             \
    }
    switch (N) {
        SSD_DECH_CASE(4) SSD_DECH_CASE(8) SSD_DECH_CASE(16) SSD_DECH_CASE(32)
        SSD_DECH_CASE(64) SSD_DECH_CASE(128) SSD_DECH_CASE(256)
        default: return cudaErrorInvalidValue;
    }
#undef SSD_DECH_CASE
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_dec_head_t(float* state, void* conv_state, const void* xBC, const float* w,
                                     const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                     const float* D, void* y, int* arrivals, int b, int H, int P, int N, int G,
                                     int k, cudaStream_t s)
{
    switch (k) {
        case 2: return launch_dec_head_k<T, 2>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, arrivals, b, H, P, N, G, s);
        case 3: return launch_dec_head_k<T, 3>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, arrivals, b, H, P, N, G, s);
        case 4: return launch_dec_head_k<T, 4>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, arrivals, b, H, P, N, G, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_step_head(float* state, void* conv_state, const void* xBC, const float* w,
                                    const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                    const float* D, void* y, int* arrivals, int b, int H, int P, int N, int G, int k,
                                    bool bf16, cudaStream_t s)
{
    return bf16 ? launch_dec_head_t<__nv_bfloat16>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y,
                                                   arrivals, b, H, P, N, G, k, s)
                : launch_dec_head_t<float>(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, arrivals, b,
                                           H, P, N, G, k, s);
}

bool state_update_supports_n(int N)
{
    return N == 4 || N == 8 || N == 16 || N == 32 || N == 64 || N == 128 || N == 256;
}

cudaError_t launch_state_update(float* state, const void* x, const void* B, const void* C,
                                int64_t row_stride, const void* dt_raw, const float* dt_bias,
                                const float* A, const float* D, void* y, int b, int H, int P,
                                int N, int G, bool bf16, cudaStream_t s)
{
    return bf16 ? launch_su_t<__nv_bfloat16>(state, x, B, C, row_stride, dt_raw, dt_bias, A, D, y,
                                             b, H, P, N, G, s)
                : launch_su_t<float>(state, x, B, C, row_stride, dt_raw, dt_bias, A, D, y, b, H,
                                     P, N, G, s);
}

}  // namespace ssd
