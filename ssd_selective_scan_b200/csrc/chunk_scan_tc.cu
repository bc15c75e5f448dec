// chunk_scan_tc.cu -- chunked SSD scan on the 5th-generation tensor cores
// (tcgen05 + TMEM), bf16 I/O, fp32 accumulation and fp32 state.
//
// The state-space duality of "Hybrid Architectures for Language Models"
// (summary page, section 2 Background: the recurrence h_t = Abar h_{t-1} +
// Bbar x_t, y_t = C h_t + D x_t recast as matrix products) evaluated in
// chunks of Q = 128 tokens (the Mamba-2 chunk size of the Nemotron feasibility
// report, sections 1.4 and 2.6).  For one (sequence, head) and one chunk,
// with dt_i = softplus(dt_raw_i + dt_bias) and cl_i = sum_{r<=i} dt_r A log2(e):
//
//   G      = C B^T                         (Q x Q, K = N)    tcgen05, TMEM
//   M[i,j] = G[i,j] 2^(cl_i - cl_j) dt_j    (j <= i, else 0)  CUDA cores -> smem
//   Yd     = M X                           (Q x P, K = Q)    tcgen05, TMEM
//   Yo     = C h_prev^T                    (Q x P, K = N)    tcgen05, TMEM
//   S^T    = B^T (w o X), w_j = 2^(cl_last - cl_j) dt_j      tcgen05, TMEM
//   h      = 2^(cl_last) h_prev + S        fp32, registers (one state column n per thread)
//   y_i    = Yd_i + 2^(cl_i) Yo_i + D x_i                    -> bf16
//
// One CTA per (sequence, head) walks the chunks in order; the fp32 state
// never leaves the chip.  B, C and X tiles arrive by TMA (128-byte swizzle,
// no multicast) straight in the layout the tensor cores read; M, w o X and
// the bf16 copy of the state are written by the threads in the same
// swizzled layouts.  Token rows past the end of the sequence are zero-filled
// by TMA and get dt = 0, so a ragged last chunk needs no special case.
//
// Every mbarrier wait is bounded (1 s); a CTA that gives up records
// SSD_ERR_TIMEOUT in the optional status word and runs to its end without
// waiting again, so a failing launch still terminates.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kQ = 128;        // chunk length
constexpr int kP = 64;         // head dim
constexpr int kN = 128;        // state size
constexpr int kThreads = 128;  // one thread per token row / state column
constexpr uint32_t kTmemCols = 256;
constexpr uint64_t kWaitNs = 1000000000ull;

// Shared-memory layout, offsets from a 1024-byte aligned base.  Tiles are
// 128-byte swizzled: 128-byte rows, 16-byte chunk c of row r at r*128 +
// ((c ^ (r & 7)) * 16).  Tiles 128 elements wide along their contiguous
// dimension are stored as two 16 KB halves (64 elements each).
constexpr int kOffB = 0;              // B tile  [128 tok][128 n]   (2 halves)
constexpr int kOffC = 32768;          // C tile  [128 tok][128 n]   (2 halves), then M [128 i][128 j]
constexpr int kOffX = 65536;          // X tile  [128 tok][64 p]
constexpr int kOffXw = 81920;         // w o X   [128 tok][64 p]
constexpr int kOffH = 98304;          // bf16 state [128 n][64 p]
constexpr int kOffCl = 114688;        // float[128] cumulative log2 decay
constexpr int kOffDt = kOffCl + 512;  // float[128] dt
constexpr int kOffWs = kOffDt + 512;  // float[4] warp totals
constexpr int kOffBar = kOffWs + 64;  // 3 mbarriers
constexpr int kOffTmem = kOffBar + 64;
constexpr int kSmemBytes = kOffTmem + 16 + 1024;   // + alignment slack

constexpr uint32_t kTileHalf = 16384;
constexpr uint32_t kLoadBytes = 2 * 32768 + 16384;

// instruction descriptors
constexpr uint32_t kIdG = umma_idesc_bf16(128, 128, false, false);   // C (K-maj) x B (K-maj)
constexpr uint32_t kIdYo = umma_idesc_bf16(128, 64, false, true);    // C (K-maj) x h (MN-maj)
constexpr uint32_t kIdYd = umma_idesc_bf16(128, 64, false, true);    // M (K-maj) x X (MN-maj)
constexpr uint32_t kIdS = umma_idesc_bf16(128, 64, true, true);      // B^T (MN-maj) x wX (MN-maj)

__device__ inline uint32_t sw128(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ inline uint4 pack_bf16x8(const float* v)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ inline void unpack_bf16x8(uint4 q, float* v)
{
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// K-major operand, 128 rows, K = 128 as two 64-wide halves: descriptor of
// K-step k (16 elements).
__device__ inline uint64_t desc_kmajor(uint32_t base, int k)
{
    return umma_desc_sw128(base + (uint32_t)(k >> 2) * kTileHalf + (uint32_t)(k & 3) * 32u, 16u, 1024u);
}

// MN-major operand with K along 128 rows: descriptor of K-step k; 64-wide
// M/N blocks are kTileHalf apart.
__device__ inline uint64_t desc_mnmajor(uint32_t base, int k)
{
    return umma_desc_sw128(base + (uint32_t)k * 2048u, kTileHalf, 1024u);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __nv_bfloat16* __restrict__ dt_raw,
                     const float* __restrict__ dt_bias, const float* __restrict__ A,
                     const float* __restrict__ D, const float* __restrict__ init_state,
                     __nv_bfloat16* __restrict__ y, float* __restrict__ final_state, int L, int H,
                     int G, int32_t* status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int aborted;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x % H;
    const int bi = blockIdx.x / H;
    const int g = h / (H / G);

    uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* bar_mma1 = bar_load + 1;
    uint64_t* bar_mma2 = bar_load + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
    float* sCl = reinterpret_cast<float*>(smem + kOffCl);
    float* sDt = reinterpret_cast<float*>(smem + kOffDt);
    float* sWs = reinterpret_cast<float*>(smem + kOffWs);
    uint8_t* sB = smem + kOffB;
    uint8_t* sC = smem + kOffC;   // C, then M
    uint8_t* sX = smem + kOffX;
    uint8_t* sXw = smem + kOffXw;
    uint8_t* sH = smem + kOffH;
    const uint32_t aB = smem_u32(sB), aC = smem_u32(sC), aX = smem_u32(sX), aXw = smem_u32(sXw),
                   aH = smem_u32(sH);

    if (tid == 0) {
        aborted = 0;
        mbar_init(bar_load, 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmC);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);

    // fp32 state: thread n holds column n of h (h[p][n], p = 0..63)
    float hs[kP];
    const size_t sbase = ((size_t)bi * H + h) * (size_t)(kP * kN);
#pragma unroll
    for (int p = 0; p < kP; ++p) hs[p] = init_state ? init_state[sbase + (size_t)p * kN + tid] : 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(sH + sw128(tid, c)) = pack_bf16x8(&hs[c * 8]);
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    const uint32_t tmem = *tmem_slot;
    const uint32_t tG = tmem;           // G, cols [0,128); then Yd [0,64) and S [64,128)
    const uint32_t tYd = tmem;
    const uint32_t tS = tmem + 64;
    const uint32_t tYo = tmem + 128;    // Yo, cols [128,192)
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    const float A2 = A[h] * 1.4426950408889634f;   // A * log2(e)
    const float Dh = D ? D[h] : 0.0f;
    const float bias = dt_bias ? dt_bias[h] : 0.0f;
    const int nchunks = (L + kQ - 1) / kQ;

    for (int c = 0; c < nchunks; ++c) {
        const uint32_t ph = (uint32_t)c & 1u;
        const int t0 = c * kQ;
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_load, kLoadBytes);
            tma_load_3d(sB, &tmB, g * kN, t0, bi, bar_load);
            tma_load_3d(sB + kTileHalf, &tmB, g * kN + 64, t0, bi, bar_load);
            tma_load_3d(sC, &tmC, g * kN, t0, bi, bar_load);
            tma_load_3d(sC + kTileHalf, &tmC, g * kN + 64, t0, bi, bar_load);
            tma_load_3d(sX, &tmX, h * kP, t0, bi, bar_load);
        }

        // dt and the inclusive cumulative log2 decay of token tid
        const int t = t0 + tid;
        float dt = 0.0f;
        if (t < L) dt = softplus_f(__bfloat162float(dt_raw[((size_t)bi * L + t) * H + h]) + bias);
        float a = dt * A2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, a, o);
            if (lane >= o) a += v;
        }
        if (lane == 31) sWs[warp] = a;
        __syncthreads();
        float pre = 0.0f;
        for (int w = 0; w < warp; ++w) pre += sWs[w];
        const float cl = a + pre;
        sCl[tid] = cl;
        sDt[tid] = dt;
        __syncthreads();
        const float cl_last = sCl[kQ - 1];

        mbar_wait_bounded(bar_load, ph, kWaitNs, &aborted, status);
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < 8; ++k)   // G = C B^T
                umma_bf16(tG, desc_kmajor(aC, k), desc_kmajor(aB, k), kIdG, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)   // Yo = C h^T
                umma_bf16(tYo, desc_kmajor(aC, k), desc_mnmajor(aH, k), kIdYo, k > 0);
            umma_commit(bar_mma1);
        }

        // w o X, row tid
        {
            const float wj = exp2f(cl_last - cl) * dt;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float v[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(sX + sw128(tid, q)), v);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] *= wj;
                *reinterpret_cast<uint4*>(sXw + sw128(tid, q)) = pack_bf16x8(v);
            }
        }

        mbar_wait_bounded(bar_mma1, ph, kWaitNs, &aborted, status);
        tc_fence_after_sync();
        // M = G o L, row tid, written over C (both MMAs reading C are done)
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            uint4 packed[4];
            if (jb <= warp) {
                float gv[32];
                tmem_ld32(tG + lane_off + jb * 32, gv);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = jb * 32 + q * 8 + e;
                        const float v = gv[q * 8 + e] * exp2f(cl - sCl[j]) * sDt[j];
                        m[e] = (j <= tid) ? v : 0.0f;
                    }
                    packed[q] = pack_bf16x8(m);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) packed[q] = make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j0 = jb * 32 + q * 8;
                *reinterpret_cast<uint4*>(sC + (j0 >> 6) * kTileHalf + sw128(tid, (j0 & 63) >> 3)) = packed[q];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int k = 0; k < 8; ++k)   // Yd = M X
                umma_bf16(tYd, desc_kmajor(aC, k), desc_mnmajor(aX, k), kIdYd, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)   // S^T = B^T (w o X)
                umma_bf16(tS, desc_mnmajor(aB, k), desc_mnmajor(aXw, k), kIdS, k > 0);
            umma_commit(bar_mma2);
        }
        mbar_wait_bounded(bar_mma2, ph, kWaitNs, &aborted, status);
        tc_fence_after_sync();

        // state: h = 2^cl_last h + S (column tid), and its bf16 copy for the next chunk
        const float decay = exp2f(cl_last);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float s[32];
            tmem_ld32(tS + lane_off + hh * 32, s);
            tmem_wait_ld();
#pragma unroll
            for (int p = 0; p < 32; ++p) hs[hh * 32 + p] = fmaf(decay, hs[hh * 32 + p], s[p]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(sH + sw128(tid, q)) = pack_bf16x8(&hs[q * 8]);

        // output: y = Yd + 2^cl Yo + D x, token row tid
        const float sc = exp2f(cl);
        __nv_bfloat16* yrow = y + (((size_t)bi * L + t) * H + h) * kP;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float yd[32], yo[32];
            tmem_ld32(tYd + lane_off + hh * 32, yd);
            tmem_ld32(tYo + lane_off + hh * 32, yo);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float xv[8], o[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(sX + sw128(tid, hh * 4 + q)), xv);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = yd[q * 8 + e] + sc * yo[q * 8 + e] + Dh * xv[e];
                if (t < L) *reinterpret_cast<uint4*>(yrow + hh * 32 + q * 8) = pack_bf16x8(o);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    }

    if (final_state) {
#pragma unroll
        for (int p = 0; p < kP; ++p) final_state[sbase + (size_t)p * kN + tid] = hs[p];
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 3-D bf16 map over a strided channel range: dim0 = channels (contiguous),
// dim1 = tokens (stride row_bytes), dim2 = sequences (stride L * row_bytes);
// box 64 channels x 128 tokens x 1, 128-byte swizzle, zero fill out of range.
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t channels, uint64_t L, uint64_t b,
                     uint64_t row_bytes)
{
    auto fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {channels, L, b};
    const cuuint64_t strides[2] = {row_bytes, row_bytes * L};
    const cuuint32_t box[3] = {64, (cuuint32_t)kQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool chunk_scan_tc_supported(const ScanArgs& a)
{
    return a.bf16 && a.P == kP && a.N == kN && a.Q == kQ;
}

cudaError_t launch_chunk_scan_tc(const ScanArgs& a, cudaStream_t s)
{
    CUtensorMap tmX, tmB, tmC;
    const uint64_t rb = (uint64_t)a.row_stride * 2;
    cudaError_t e;
    if ((e = make_map(&tmX, a.x, (uint64_t)a.H * a.P, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = make_map(&tmB, a.B, (uint64_t)a.G * a.N, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = make_map(&tmC, a.C, (uint64_t)a.G * a.N, a.L, a.b, rb)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((int64_t)a.b * a.H));
    chunk_scan_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(
        tmX, tmB, tmC, static_cast<const __nv_bfloat16*>(a.dt_raw), a.dt_bias, a.A, a.D, a.init_state,
        static_cast<__nv_bfloat16*>(a.y), a.final_state, a.L, a.H, a.G, a.status);
    return cudaGetLastError();
}

}  // namespace ssd
