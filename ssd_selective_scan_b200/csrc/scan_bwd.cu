// scan_bwd.cu -- backward pass of the chunked SSD scan (gradients for
// training; the Nemotron feasibility report plans forward and backward tests
// of the Mamba-2 layer, sections 3.2 and 3.3).
//
// The forward is the recurrence of "Hybrid Architectures for Language
// Models" (summary page, section 2 Background), h_t = exp(dt_t A) h_{t-1} +
// dt_t x_t B_t^T, y_t = h_t C_t + D x_t, dt = softplus(dt_raw + dt_bias).
// Given dy and the final state's gradient dfinal, this computes dx, dB, dC,
// ddt_raw, dA, dD, ddt_bias and the initial state's gradient, chunk by chunk
// in matrix form (state-space duality applied to the gradient).  For a chunk
// with entering state h0 and incoming state gradient g_end, cum = inclusive
// cumsum of dt A inside the chunk and Lm[i][j] = exp(cum_i - cum_j), j <= i:
//   dC_i  = e^cum_i (dY h0)_i + sum_{j<=i} Lm[i][j] dt_j (dy_i.x_j) B_j
//   gB_j  = e^(cum_last-cum_j) (B_j g_end^T) + sum_{k>=j} Lm[k][j] (C_k.B_j) dy_k
//   U_j   = e^(cum_last-cum_j) (x_j^T g_end) + sum_{k>=j} Lm[k][j] (dy_k.x_j) C_k
//   dx_j  = D dy_j + dt_j gB_j,   dB_j = dt_j U_j,   ddt_j = U_j.B_j + A r_j
//   r_t   = <g_t, exp(dt_t A) h_{t-1}>
//         = e^cum_last <g_end, h0> + sum_{j<=t} e^(cum_last-cum_j) dt_j x_j^T g_end B_j
//           + sum_{k>=t} e^cum_k dy_k^T h0 C_k + sum_{k>=t, j<=t} W[k][j] - dt_t U_t.B_t,
//   W[k][j] = Lm[k][j] dt_j (dy_k.x_j)(C_k.B_j)
//   dA += sum_t dt_t r_t,  ddt_raw = ddt sigmoid(dt_raw + dt_bias)
// and the entering state's gradient e^cum_last g_end + sum_k e^cum_k dy_k C_k^T
// becomes the previous chunk's g_end.
//
// General path, float32 arithmetic on the CUDA cores: one CTA per (sequence,
// head) walks the chunks forward (storing each chunk's entering state in the
// workspace), then backward.  Each phase of a chunk is a loop over output
// elements, `for (i = tid; i < n; i += nthreads)`, between barriers.  dB and
// dC of each head, and the per-(sequence, head) sums of dA, dD and ddt_bias,
// go to the workspace; a second kernel adds them over the heads of a group
// and over the batch in a fixed order, so the result is deterministic.
#include <algorithm>

#include "common.cuh"
#include "scan_bwd.h"

namespace ssd {

namespace {

template <typename T>
__device__ inline void store_f(T* p, float v) { *p = io<T>::from_f(v); }

constexpr int kBwdThreads = 1024;
constexpr int kBwdQ = 32;   // chunk length of the backward pass

struct BwdParams {
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
    void* ddt_raw;
    float* dinit;
    float* ws_h0;     // [b*H][chunks][P][N]
    float* ws_dB;     // [b][L][H][N]
    float* ws_dC;     // [b][L][H][N]
    float* ws_part;   // [3][b*H]: dA, dD, ddt_bias per (sequence, head)
    int L, H, P, N, G;
};

// Shared-memory rows are padded by one float (row strides P+1, N+1, Q+1):
// the phases that give each lane of a warp its own row (the Gram tiles, dx,
// the per-token scalars) then hit 32 different banks instead of one.
__host__ __device__ inline int bwd_smem_floats(int P, int N)
{
    const int Q = kBwdQ, PS = P + 1, NS = N + 1, QS = Q + 1;
    return 2 * P * NS + 2 * Q * PS + 2 * Q * NS + 3 * Q * QS + 3 * Q * NS + 15 * Q + kBwdThreads / 32;
}

__device__ inline float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
scan_bwd_chain_kernel(const BwdParams p)
{
    extern __shared__ float sm[];
    const int P = p.P, N = p.N, L = p.L, H = p.H;
    const int Q = kBwdQ, PS = P + 1, NS = N + 1, QS = Q + 1;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
    const int chain = blockIdx.x;
    const int bi = chain / H, h = chain - bi * H;
    const int grp = h / (H / p.G);
    const int nchunks = (L + Q - 1) / Q;

    float* sH0 = sm;                 // [P][NS] entering state of the chunk
    float* sG = sH0 + P * NS;        // [P][NS] state gradient at the chunk's end
    float* sX = sG + P * NS;         // [Q][PS]
    float* sDY = sX + Q * PS;        // [Q][PS]
    float* sB = sDY + Q * PS;        // [Q][NS]
    float* sC = sB + Q * NS;         // [Q][NS]
    float* sYX = sC + Q * NS;        // [Q][QS] dy_i . x_j
    float* sCB = sYX + Q * QS;       // [Q][QS] C_i . B_j
    float* sLm = sCB + Q * QS;       // [Q][QS] exp(cum_i - cum_j), j <= i (else 0)
    float* sT1 = sLm + Q * QS;       // [Q][NS] dY h0
    float* sT2 = sT1 + Q * NS;       // [Q][NS] X g_end
    float* sU = sT2 + Q * NS;        // [Q][NS] U
    float* sDt = sU + Q * NS;        // [Q]
    float* sCum = sDt + Q;           // [Q] inclusive cumsum of dt A
    float* sSig = sCum + Q;          // [Q] sigmoid(dt_raw + dt_bias)
    float* sXgB = sSig + Q;          // [Q] x_j^T g_end B_j
    float* sYhC = sXgB + Q;          // [Q] dy_k^T h0 C_k
    float* sUB = sYhC + Q;           // [Q] U_j . B_j
    float* sCol = sUB + Q;           // [Q] sum_{k>=t} W[k][t]
    float* sRow = sCol + Q;          // [Q] sum_{j<=t} W[t][j]
    float* sDD = sRow + Q;           // [Q] dy_t . x_t
    float* sEl = sDD + Q;            // [Q] exp(cum_last - cum_j) (times dt_j in the forward sweep)
    float* sEc = sEl + Q;            // [Q] exp(cum_j)
    float* sE = sEc + Q;             // [1]: exp(cum_last)
    float* sMisc = sE + Q;           // [3 Q]: scratch of the sequential step
    float* sRed = sMisc + 3 * Q;     // [nwarps] block reduction

    const T* xg = static_cast<const T*>(p.x);
    const T* Bg = static_cast<const T*>(p.B);
    const T* Cg = static_cast<const T*>(p.C);
    const T* dtr = static_cast<const T*>(p.dt_raw);
    const T* dyg = static_cast<const T*>(p.dy);
    const float A = p.A[h];
    const float Dh = p.D ? p.D[h] : 0.0f;
    const float dtb = p.dt_bias ? p.dt_bias[h] : 0.0f;
    const size_t tok0 = (size_t)bi * L;
    float* h0s = p.ws_h0 + (size_t)chain * nchunks * P * N;

    // chunk c's token inputs into shared memory, dt, its cumulative decay
    auto load_chunk = [&](int c, bool with_dy) {
        const int s0 = c * Q, q = min(Q, L - s0);
        for (int i = tid; i < Q * P; i += nt) {
            const int j = i / P, pp = i - j * P;
            const size_t t = tok0 + s0 + j;
            sX[j * PS + pp] = j < q ? ld_f(xg + t * p.row_stride + (size_t)h * P + pp) : 0.0f;
            if (with_dy) sDY[j * PS + pp] = j < q ? ld_f(dyg + (t * H + h) * P + pp) : 0.0f;
        }
        for (int i = tid; i < Q * N; i += nt) {
            const int j = i / N, n = i - j * N;
            const size_t t = tok0 + s0 + j;
            sB[j * NS + n] = j < q ? ld_f(Bg + t * p.row_stride + (size_t)grp * N + n) : 0.0f;
            if (with_dy) sC[j * NS + n] = j < q ? ld_f(Cg + t * p.row_stride + (size_t)grp * N + n) : 0.0f;
        }
        for (int j = tid; j < Q; j += nt) {
            const float v = j < q ? ld_f(dtr + (tok0 + s0 + j) * H + h) + dtb : 0.0f;
            sDt[j] = j < q ? softplus_f(v) : 0.0f;
            sSig[j] = 1.0f / (1.0f + expf(-v));
        }
        __syncthreads();
        if (tid == 0) {
            float run = 0.0f;
            for (int j = 0; j < Q; ++j) {
                run += sDt[j] * A;
                sCum[j] = run;
            }
        }
        __syncthreads();
        return q;
    };

    // ---------------- forward: the state entering every chunk ----------------
    for (int i = tid; i < P * N; i += nt) {
        const int pp = i / N, n = i - pp * N;
        sH0[pp * NS + n] = p.init_state ? p.init_state[(size_t)chain * P * N + i] : 0.0f;
    }
    __syncthreads();
    for (int c = 0; c < nchunks; ++c) {
        for (int i = tid; i < P * N; i += nt) {
            const int pp = i / N, n = i - pp * N;
            h0s[(size_t)c * P * N + i] = sH0[pp * NS + n];
        }
        const int q = load_chunk(c, false);
        const float cl = sCum[q - 1];
        for (int j = tid; j < Q; j += nt) sEl[j] = j < q ? expf(cl - sCum[j]) * sDt[j] : 0.0f;
        __syncthreads();
        const float ecl = expf(cl);
        for (int i = tid; i < P * N; i += nt) {
            const int pp = i / N, n = i - pp * N;
            float acc = ecl * sH0[pp * NS + n];
            for (int j = 0; j < q; ++j) acc += sX[j * PS + pp] * sEl[j] * sB[j * NS + n];
            sH0[pp * NS + n] = acc;
        }
        __syncthreads();
    }

    // ---------------- backward over the chunks ----------------
    for (int i = tid; i < P * N; i += nt) {
        const int pp = i / N, n = i - pp * N;
        sG[pp * NS + n] = p.dfinal ? p.dfinal[(size_t)chain * P * N + i] : 0.0f;
    }
    float accA = 0.0f, accD = 0.0f, accBias = 0.0f;   // thread 0's sums
    for (int c = nchunks - 1; c >= 0; --c) {
        const int s0 = c * Q;
        for (int i = tid; i < P * N; i += nt) {
            const int pp = i / N, n = i - pp * N;
            sH0[pp * NS + n] = h0s[(size_t)c * P * N + i];
        }
        const int q = load_chunk(c, true);
        const float cl = sCum[q - 1];

        // 1. the chunk's Gram tiles and the products with h0 and g_end
        for (int i = tid; i < Q * Q; i += nt) {
            const int a = i / Q, bb = i - a * Q;
            float yx = 0.0f, cb = 0.0f;
            for (int pp = 0; pp < P; ++pp) yx += sDY[a * PS + pp] * sX[bb * PS + pp];
            for (int n = 0; n < N; ++n) cb += sC[a * NS + n] * sB[bb * NS + n];
            sYX[a * QS + bb] = yx;
            sCB[a * QS + bb] = cb;
            sLm[a * QS + bb] = (bb <= a && a < q) ? expf(sCum[a] - sCum[bb]) : 0.0f;
        }
        for (int j = tid; j < Q; j += nt) {
            sEl[j] = j < q ? expf(cl - sCum[j]) : 0.0f;
            sEc[j] = j < q ? expf(sCum[j]) : 0.0f;
        }
        if (tid == 0) sE[0] = expf(cl);
        for (int i = tid; i < Q * N; i += nt) {
            const int k = i / N, n = i - k * N;
            float t1 = 0.0f, t2 = 0.0f;
            for (int pp = 0; pp < P; ++pp) {
                t1 += sDY[k * PS + pp] * sH0[pp * NS + n];
                t2 += sX[k * PS + pp] * sG[pp * NS + n];
            }
            sT1[k * NS + n] = t1;
            sT2[k * NS + n] = t2;
        }
        // <g_end, h0>: per-thread partials, then one per warp
        {
            float part = 0.0f;
            for (int i = tid; i < P * N; i += nt) {
                const int pp = i / N, n = i - pp * N;
                part += sG[pp * NS + n] * sH0[pp * NS + n];
            }
            part = warp_sum(part);
            if (lane == 0) sRed[warp] = part;
        }
        __syncthreads();

        // 2. dC and U (token rows x N), dx (token rows x P)
        for (int i = tid; i < Q * N; i += nt) {
            const int r = i / N, n = i - r * N;
            float dc = 0.0f, u = 0.0f;
            if (r < q) {
                dc = sEc[r] * sT1[r * NS + n];
                for (int j = 0; j <= r; ++j) dc += sLm[r * QS + j] * sDt[j] * sYX[r * QS + j] * sB[j * NS + n];
                u = sEl[r] * sT2[r * NS + n];
                for (int k = r; k < q; ++k) u += sLm[k * QS + r] * sYX[k * QS + r] * sC[k * NS + n];
                const size_t t = tok0 + s0 + r;
                p.ws_dC[(t * H + h) * N + n] = dc;
                p.ws_dB[(t * H + h) * N + n] = sDt[r] * u;
            }
            sU[r * NS + n] = u;
        }
        for (int i = tid; i < Q * P; i += nt) {
            const int j = i / P, pp = i - j * P;
            if (j < q) {
                float gb = 0.0f;
                for (int n = 0; n < N; ++n) gb += sB[j * NS + n] * sG[pp * NS + n];
                gb *= sEl[j];
                for (int k = j; k < q; ++k) gb += sLm[k * QS + j] * sCB[k * QS + j] * sDY[k * PS + pp];
                const float dxv = Dh * sDY[j * PS + pp] + sDt[j] * gb;
                store_f(static_cast<T*>(p.dx) + ((tok0 + s0 + j) * H + h) * P + pp, dxv);
            }
        }
        __syncthreads();

        // 3. per-token scalars, one warp per token: x^T g_end B, dy^T h0 C,
        //    U.B, dy.x, the masked pair tile's column and row sums
        for (int j = warp; j < Q; j += nwarps) {
            float xgb = 0.0f, yhc = 0.0f, ub = 0.0f, dd = 0.0f, col = 0.0f, row = 0.0f;
            if (j < q) {
                for (int n = lane; n < N; n += 32) {
                    const float b = sB[j * NS + n];
                    xgb += sT2[j * NS + n] * b;
                    yhc += sT1[j * NS + n] * sC[j * NS + n];
                    ub += sU[j * NS + n] * b;
                }
                for (int pp = lane; pp < P; pp += 32) dd += sDY[j * PS + pp] * sX[j * PS + pp];
                for (int k = j + lane; k < q; k += 32)   // W[k][j], k >= j
                    col += sLm[k * QS + j] * sDt[j] * sYX[k * QS + j] * sCB[k * QS + j];
                for (int i2 = lane; i2 <= j; i2 += 32)   // W[j][i2], i2 <= j
                    row += sLm[j * QS + i2] * sDt[i2] * sYX[j * QS + i2] * sCB[j * QS + i2];
            }
            xgb = warp_sum(xgb);
            yhc = warp_sum(yhc);
            ub = warp_sum(ub);
            dd = warp_sum(dd);
            col = warp_sum(col);
            row = warp_sum(row);
            if (lane == 0) {
                sXgB[j] = xgb;
                sYhC[j] = yhc;
                sUB[j] = ub;
                sDD[j] = dd;
                sCol[j] = col;
                sRow[j] = row;
            }
        }
        __syncthreads();

        // 4. the decay gradient and ddt (sequential over the chunk's tokens)
        if (tid == 0) {
            float gh0 = 0.0f;
            for (int w = 0; w < nwarps; ++w) gh0 += sRed[w];
            const float t1 = sE[0] * gh0;
            float* t3 = sMisc;   // suffix sums of e^cum_k dy_k^T h0 C_k
            float suf = 0.0f;
            for (int k = q - 1; k >= 0; --k) {
                suf += sEc[k] * sYhC[k];
                t3[k] = suf;
            }
            float t2 = 0.0f, S = 0.0f;
            for (int t = 0; t < q; ++t) {
                t2 += sEl[t] * sDt[t] * sXgB[t];
                S += sCol[t] - (t > 0 ? sRow[t - 1] : 0.0f);
                const float r = t1 + t2 + t3[t] + S - sDt[t] * sUB[t];
                const float ddt = sUB[t] + A * r;
                const float dv = ddt * sSig[t];
                store_f(static_cast<T*>(p.ddt_raw) + (tok0 + s0 + t) * H + h, dv);
                accA += sDt[t] * r;
                accD += sDD[t];
                accBias += dv;
            }
        }
        // 5. the entering state's gradient, the previous chunk's g_end
        for (int i = tid; i < P * N; i += nt) {
            const int pp = i / N, n = i - pp * N;
            float g = sE[0] * sG[pp * NS + n];
            for (int k = 0; k < q; ++k) g += sEc[k] * sDY[k * PS + pp] * sC[k * NS + n];
            sG[pp * NS + n] = g;
        }
        __syncthreads();
    }
    if (p.dinit)
        for (int i = tid; i < P * N; i += nt) {
            const int pp = i / N, n = i - pp * N;
            p.dinit[(size_t)chain * P * N + i] = sG[pp * NS + n];
        }
    if (tid == 0) {
        const int nch = (int)gridDim.x;
        p.ws_part[chain] = accA;
        p.ws_part[nch + chain] = accD;
        p.ws_part[2 * nch + chain] = accBias;
    }
}

// dB, dC [b][L][G][N] = sum over the group's heads, in head order
template <typename T>
__global__ void scan_bwd_group_sum_kernel(const float* __restrict__ ws_dB, const float* __restrict__ ws_dC,
                                          T* __restrict__ dB, T* __restrict__ dC, int64_t rows, int H, int G,
                                          int N)
{
    const int hpg = H / G;
    const int64_t total = rows * G * N;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / ((int64_t)G * N);
        const int rem = (int)(i - t * G * N);
        const int g = rem / N, n = rem - g * N;
        float sb = 0.0f, sc = 0.0f;
        for (int k = 0; k < hpg; ++k) {
            const int64_t src = (t * H + g * hpg + k) * N + n;
            sb += ws_dB[src];
            sc += ws_dC[src];
        }
        store_f(dB + i, sb);
        store_f(dC + i, sc);
    }
}

// dA, dD, ddt_bias [H] = sum over the batch, in batch order
__global__ void scan_bwd_head_sum_kernel(const float* __restrict__ part, float* __restrict__ dA,
                                         float* __restrict__ dD, float* __restrict__ dbias, int b, int H)
{
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    const int nch = b * H;
    float a = 0.0f, d = 0.0f, s = 0.0f;
    for (int bi = 0; bi < b; ++bi) {
        a += part[bi * H + h];
        d += part[nch + bi * H + h];
        s += part[2 * nch + bi * H + h];
    }
    dA[h] = a;
    dD[h] = d;
    dbias[h] = s;
}

size_t align256(size_t n) { return (n + 255) / 256 * 256; }

}  // namespace

size_t scan_bwd_smem_bytes(int P, int N) { return (size_t)bwd_smem_floats(P, N) * 4; }

size_t scan_bwd_workspace_bytes(int b, int L, int H, int P, int N)
{
    if (b <= 0 || L <= 0) return 0;
    const size_t chains = (size_t)b * H;
    const size_t nchunks = (size_t)(L + kBwdQ - 1) / kBwdQ;
    return align256(chains * nchunks * P * N * 4) + 2 * align256((size_t)b * L * H * N * 4) +
           align256(3 * chains * 4);
}

cudaError_t launch_scan_bwd(const ScanBwdArgs& a, cudaStream_t s)
{
    BwdParams p;
    p.x = a.x;
    p.B = a.B;
    p.C = a.C;
    p.row_stride = a.row_stride;
    p.dt_raw = a.dt_raw;
    p.dt_bias = a.dt_bias;
    p.A = a.A;
    p.D = a.D;
    p.init_state = a.init_state;
    p.dy = a.dy;
    p.dfinal = a.dfinal;
    p.dx = a.dx;
    p.ddt_raw = a.ddt_raw;
    p.dinit = a.dinit;
    p.L = a.L;
    p.H = a.H;
    p.P = a.P;
    p.N = a.N;
    p.G = a.G;
    const size_t chains = (size_t)a.b * a.H;
    const size_t nchunks = (size_t)(a.L + kBwdQ - 1) / kBwdQ;
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    p.ws_h0 = reinterpret_cast<float*>(ws);
    ws += align256(chains * nchunks * a.P * a.N * 4);
    p.ws_dB = reinterpret_cast<float*>(ws);
    ws += align256((size_t)a.b * a.L * a.H * a.N * 4);
    p.ws_dC = reinterpret_cast<float*>(ws);
    ws += align256((size_t)a.b * a.L * a.H * a.N * 4);
    p.ws_part = reinterpret_cast<float*>(ws);

    const size_t smem = scan_bwd_smem_bytes(a.P, a.N);
    const int64_t rows = (int64_t)a.b * a.L;
    const int64_t total = rows * a.G * a.N;
    const int sum_blocks = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
    if (a.bf16) {
        auto k = scan_bwd_chain_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<(unsigned)chains, kBwdThreads, smem, s>>>(p);
        scan_bwd_group_sum_kernel<__nv_bfloat16><<<sum_blocks, 256, 0, s>>>(
            p.ws_dB, p.ws_dC, static_cast<__nv_bfloat16*>(a.dB), static_cast<__nv_bfloat16*>(a.dC), rows, a.H, a.G,
            a.N);
    } else {
        auto k = scan_bwd_chain_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<(unsigned)chains, kBwdThreads, smem, s>>>(p);
        scan_bwd_group_sum_kernel<float><<<sum_blocks, 256, 0, s>>>(p.ws_dB, p.ws_dC, static_cast<float*>(a.dB),
                                                                    static_cast<float*>(a.dC), rows, a.H, a.G, a.N);
    }
    scan_bwd_head_sum_kernel<<<(a.H + 127) / 128, 128, 0, s>>>(p.ws_part, a.dA, a.dD, a.ddt_bias, a.b, a.H);
    return cudaGetLastError();
}

}  // namespace ssd
