// gemm_tc.cu -- the Mamba-2 mixer's projections on the 5th-generation tensor
// cores: C[M][N] = A[M][K] B[N][K]^T with bf16 operands, fp32 accumulation in
// TMEM and bf16 output (in_proj: hidden x W_in^T; out_proj: normed y x
// W_out^T -- the linear layers of the Nemotron feasibility report, section
// 3.3, around the bf16/fp32 scan).
//
// Persistent, warp-specialized, one CTA per SM:
//   warp 0  (one thread)   TMA loads of A (128 x 64) and B (256 x 64) tiles,
//                          128-byte swizzle, into a ring of kStages stages;
//   warp 1  (one thread)   tcgen05.mma M128 N256 K16, four per stage, into
//                          one of two TMEM accumulators (256 columns each);
//   warps 2-5              the epilogue: TMEM -> registers -> bf16 -> global,
//                          one TMEM lane quadrant (32 rows) per warp, while
//                          the MMA warp fills the other accumulator.
// Tiles are walked n-fastest (all N tiles of one row block of A in turn), so
// an A row block is read from HBM once and B, the weights, stays in L2.
// An optional column split sends output columns >= n_split to a second
// matrix (in_proj: z | xBC to one buffer, dt to another); n_split is a
// multiple of 8.  Every wait is bounded (1 s) and reports
// SSD_ERR_TIMEOUT in the optional status word.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB
constexpr int kBBytes = kBN * kBK * 2;          // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;  // 48 KB
constexpr int kGemmThreads = 192;               // 6 warps
constexpr int kEpiWarps = 4;
constexpr uint32_t kAccCols = 256;              // fp32 columns per accumulator
constexpr uint64_t kGemmWaitNs = 1000000000ull;
constexpr int kOffBars = kStages * kStageBytes;               // full[S], empty[S], tfull[2], tempty[2]
constexpr int kGemmSmem = kOffBars + 8 * (2 * kStages + 4) + 16 + 1024;

constexpr uint32_t kIdesc = umma_idesc_bf16(kBM, kBN, false, false);   // both operands K-major

struct GemmParams {
    int M, N, K;
    int n_split;                 // columns >= n_split go to C1 (0: none)
    __nv_bfloat16* C0;
    int64_t ldc0;
    __nv_bfloat16* C1;
    int64_t ldc1;
    int tiles_m, tiles_n;
    int32_t* status;
};

// K-major operand of `rows` rows, 128-byte swizzle: descriptor of K step kk
// (16 elements) within a 64-wide K tile.
__device__ inline uint64_t desc_k(uint32_t base, int kk) { return umma_desc_sw128(base + (uint32_t)kk * 32u, 16u, 1024u); }

__device__ inline void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const GemmParams prm)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBars);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;    // [2] accumulator ready (MMA commit)
    uint64_t* tempty = tfull + 2;         // [2] accumulator drained (epilogue warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* aborted = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = prm.tiles_m * prm.tiles_n;
    const int ksteps = (prm.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        *aborted = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, kEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 2 * kAccCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
            int it = 0;   // stage counter over all tiles
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
                const int mb = t / prm.tiles_n, nb = t - mb * prm.tiles_n;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    // the stage was consumed by the MMAs of use it - kStages
                    if (it >= kStages) mbar_wait_bounded(empty + s, ph ^ 1u, kGemmWaitNs, aborted, prm.status);
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(full + s, kStageBytes);
                    tma_load_2d(st, &tmA, ks * kBK, mb * kBM, full + s);
                    tma_load_2d(st + kABytes, &tmB, ks * kBK, nb * kBN, full + s);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            int it = 0, local = 0;
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
                const int acc = local & 1;
                const uint32_t aph = (uint32_t)(local >> 1) & 1u;
                // the epilogue drained this accumulator (use local - 2)
                if (local >= 2) mbar_wait_bounded(tempty + acc, aph ^ 1u, kGemmWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                const uint32_t d = tmem + (uint32_t)acc * kAccCols;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    mbar_wait_bounded(full + s, ph, kGemmWaitNs, aborted, prm.status);
                    tc_fence_after_sync();
                    const uint32_t a = smem_u32(smem + s * kStageBytes);
                    const uint32_t b = a + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(d, desc_k(a, kk), desc_k(b, kk), kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(empty + s);   // the stage is free once these MMAs are done
                }
                umma_commit(tfull + acc);     // the tile's accumulator is complete
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;            // TMEM lane quadrant of this warp
        const int row_in_tile = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        int local = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
            const int mb = t / prm.tiles_n, nb = t - mb * prm.tiles_n;
            const int acc = local & 1;
            mbar_wait_bounded(tfull + acc, (uint32_t)(local >> 1) & 1u, kGemmWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            const int m = mb * kBM + row_in_tile;
            const int n0 = nb * kBN;
            const int split = prm.n_split > 0 ? prm.n_split : prm.N;
            __nv_bfloat16* const row0 = prm.C0 + (int64_t)m * prm.ldc0;
            __nv_bfloat16* const row1 = prm.C1 + (int64_t)m * prm.ldc1 - split;
            const uint32_t tbase = tmem + (uint32_t)acc * kAccCols + lane_off;
#pragma unroll 1
            for (int c = 0; c < kBN; c += 32) {
                float v[32];
                tmem_ld32(tbase + (uint32_t)c, v);
                tmem_wait_ld();
                if (m < prm.M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        // 8 columns at a time; N and n_split are multiples of 8
                        const int col = n0 + c + q * 8;
                        if (col < prm.N) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
                                w[e] = *reinterpret_cast<uint32_t*>(&h2);
                            }
                            __nv_bfloat16* dst = col < split ? row0 + col : row1 + col;
                            *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);   // the accumulator may be refilled
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 2 * kAccCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
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

// 2-D bf16 map over a row-major [rows][cols] matrix with row stride ld
// elements: box 64 columns (128 bytes) x box_rows rows, 128-byte swizzle,
// zero fill past the edges.
cudaError_t make_map2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool gemm_bf16_tn_supported(int M, int N, int K, int64_t lda, int64_t ldb, int n_split)
{
    if (M <= 0 || N <= 0 || K <= 0) return false;
    if (N % 8 || K % 8 || lda % 8 || ldb % 8 || lda < K || ldb < K) return false;
    if (n_split < 0 || n_split >= N || n_split % 8) return false;
    return true;
}

cudaError_t launch_gemm_bf16_tn(const void* A, int64_t lda, const void* B, int64_t ldb, void* C0, int64_t ldc0,
                                void* C1, int64_t ldc1, int M, int N, int K, int n_split, int32_t* status,
                                cudaStream_t s)
{
    CUtensorMap tmA, tmB;
    cudaError_t e;
    if ((e = make_map2d(&tmA, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda, kBM)) != cudaSuccess) return e;
    if ((e = make_map2d(&tmB, B, (uint64_t)K, (uint64_t)N, (uint64_t)ldb, kBN)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        sms = 148;
    GemmParams p;
    p.M = M;
    p.N = N;
    p.K = K;
    p.n_split = n_split;
    p.C0 = static_cast<__nv_bfloat16*>(C0);
    p.ldc0 = ldc0;
    p.C1 = static_cast<__nv_bfloat16*>(C1);
    p.ldc1 = ldc1;
    p.tiles_m = (M + kBM - 1) / kBM;
    p.tiles_n = (N + kBN - 1) / kBN;
    p.status = status;
    const int ntiles = p.tiles_m * p.tiles_n;
    const int grid = ntiles < sms ? ntiles : sms;
    gemm_bf16_tn_kernel<<<grid, kGemmThreads, kGemmSmem, s>>>(tmA, tmB, p);
    return cudaGetLastError();
}

}  // namespace ssd
