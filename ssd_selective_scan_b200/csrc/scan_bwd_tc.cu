// scan_bwd_tc.cu -- backward pass of the chunked SSD scan on the 5th-
// generation tensor cores (tcgen05 + TMEM): bf16 I/O, fp32 accumulation,
// chunks of Q = 128 tokens, head dim P = 64, state size N = 128.
//
// The gradients of the recurrence of "Hybrid Architectures for Language
// Models" (summary page, section 2 Background: h_t = exp(dt_t A) h_{t-1} +
// dt_t x_t B_t^T, y_t = h_t C_t + D x_t) in the chunked matrix form of
// scan_bwd.cu, reorganised so that each chunk is independent once its
// entering state h0 and the state gradient at its end g are known.  In log2
// units, l_t = dt_t A log2(e), cum = inclusive cumsum of l inside a chunk, cl
// its last value, Ec_k = 2^cum_k, El_j = 2^(cl - cum_j), Lm[i][j] =
// 2^(cum_i - cum_j) for j <= i (else 0):
//
// 1. bwd_states_kernel (tensor cores), per chunk and head:
//      S^T  = B^T (w o X),  w_j = El_j dt_j      the chunk's own end state
//      dS^T = C^T (Ec o dY)                     its part of the entering
//                                               state's gradient
// 2. bwd_pass_kernel (CUDA cores), per (sequence, head), chunk after chunk,
//    the two directions independently (fp32 sums of bf16 S and dS):
//      h0_{c+1} = 2^cl_c h0_c + S_c,   g_{c-1} = 2^cl_c g_c + dS_c;
//    the initial state's gradient is g_{-1}.
// 3. bwd_chunk_kernel (tensor cores), per chunk and head:
//      YX = dY X^T,  CB = C B^T                              (Q x Q)
//      M2 = Lm o YX,  M1 = dt_j o M2,  M3 = Lm o CB           (M1, M3 bf16 tiles)
//      dC = (Ec o dY) h0 + M1 B                              (Q x N)
//      dB = dt o U = (dt o El o X) g + M1^T C                (Q x N)
//      gB = El o (B g^T) + M3^T dY, dx = D dy + dt o gB       (Q x P)
//    and, in fp32, U_j.B_j = El_j x_j.(B g^T)_j + sum_k M2[k][j] CB[k][j].
//    With t1 = 2^cl <g, h0> (from the bf16 tiles of h0 and g), the decay
//    gradient r_t = <g_t, exp(dt_t A) h_{t-1}> has a closed form in the
//    tiles' sums (dt_j U_j.B_j = dt_j El_j x_j^T g B_j + sum_k W[k][j] and
//    dC_k.C_k = Ec_k dy_k^T h0 C_k + sum_j W[k][j], W = M1 o CB):
//      r_t = t1 - sum W + sum_{j<t} dt_j U_j.B_j + sum_{k>=t} dC_k.C_k,
//    then ddt = U.B + A r, ddt_raw = ddt sigmoid(dt_raw + dt_bias),
//    dA = sum dt r, dD = sum dy.x, ddt_bias = sum ddt_raw.  dC takes M1
//    rounded to bf16 while W is summed in fp32, so that rounding is taken
//    out exactly: dC_k.C_k - sum_j (bf16(M1) - M1)[k][j] CB[k][j].  (Without
//    it the large sums of the closed form amplify the rounding.)
// dB and dC of a group are sums over its heads: one CTA takes the heads of a
// group in order and its accumulators run on across them in TMEM.  dA, dD
// and ddt_bias are summed over sequences, chunks and row quarters in a
// fixed order by a last kernel, so the result is deterministic.
//
// Kernels 1 and 3: one CTA per (chunk, sequence, group), a TMA producer
// warp, an MMA warp (one thread issues tcgen05.mma; TMEM allocation) and
// elementwise warps that serve TMEM lanes 32*(warp%4).. (token rows, or
// state columns n).  Tiles are 128-byte swizzled, loaded by TMA without
// multicast; kernel 1 writes its bf16 state tiles by TMA store.  In kernel
// 3 the next head's loads start once the current head's products are done,
// and a head's per-token step runs while the next head's second products
// are on the tensor cores.  Every mbarrier wait is bounded (1 s); a CTA that
// gives up sets the timeout flag in the workspace's first word and ends.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "scan_bwd.h"
#include "sm100.cuh"

namespace ssd {

namespace {

using namespace sm100;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr uint32_t kTileHalf = 16384;        // 128 rows x 64 bf16, swizzled
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPassSlices = 8;               // CTAs per chain and direction in the passing kernel
constexpr int kPassThreads = 256;            // 4 state elements per thread
constexpr int kParts = 4;                    // dA / dD / ddt_bias partials per (chain, chunk)
constexpr int kMaxHpg = 256;                 // heads per group (per-head scalars kept in shared memory)

constexpr uint32_t kStatesDim = kN * kP;     // floats of one chunk state

__device__ inline uint32_t sw128(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ inline uint4 pack8(const float* v)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ inline void unpack8(uint4 q, float* v)
{
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// K-major operand, 128 rows, K up to 128 as 64-wide halves: K-step k (16 elements)
__device__ inline uint64_t desc_k(uint32_t base, int k)
{
    return umma_desc_sw128(base + (uint32_t)(k >> 2) * kTileHalf + (uint32_t)(k & 3) * 32u, 16u, 1024u);
}

// MN-major operand with K along rows: K-step k (16 rows); 64-wide M/N blocks kTileHalf apart
__device__ inline uint64_t desc_mn(uint32_t base, int k)
{
    return umma_desc_sw128(base + (uint32_t)k * 2048u, kTileHalf, 1024u);
}

// A wait that ignores the abort flag: used once at the end to let this
// CTA's own TMA loads land before shared memory is released.
__device__ inline void drain_wait(uint64_t* bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitNs) break;
}

// Named barrier among n threads that also ORs a flag over them: every
// participant gets the same answer, so a give-up seen by any thread ends
// the loop of all of them at the same barrier.
__device__ inline bool named_bar_any(int id, int n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "barrier.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ inline float warp_incl_scan(float v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Column sums over a warp's 32 rows of 16 values per lane: lane l (and
// l + 16) receives the sum of column l & 15 (31 shuffles, fixed order).
__device__ inline float warp_colsum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], 16);
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < off; ++k) {
            const float send = up ? v[k] : v[k + off];
            const float keep = up ? v[k + off] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

__device__ inline float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

__device__ inline float warp_total(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

struct TcParams {
    const __nv_bfloat16* dt_raw;   // [b][L][H]
    const __nv_bfloat16* dy;       // [b][L][H][P]
    const __nv_bfloat16* x;        // token rows row_stride apart
    int64_t row_stride;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;       // [b][H][P][N]
    const float* dfinal;           // [b][H][P][N]
    __nv_bfloat16* dx;             // [b][L][H][P]
    __nv_bfloat16* dB;             // [b][L][G][N]
    __nv_bfloat16* dC;
    __nv_bfloat16* ddt_raw;        // [b][L][H]
    float* dA;
    float* dD;
    float* ddt_bias;
    float* dinit;                  // [b][H][P][N]
    int32_t* status;               // workspace word 0: timeout flag
    __nv_bfloat16* ws_S;           // [chains][nc][N][P] bf16 S
    __nv_bfloat16* ws_dS;          // [chains][nc][N][P] bf16 dS
    __nv_bfloat16* ws_hb;          // [chains][nc][N][P] bf16 h0
    __nv_bfloat16* ws_gb;          // [chains][nc][N][P] bf16 g
    float* ws_cl;                  // [chains][nc]
    float* ws_part;                // [3][chains][nc][kParts]
    int b, L, H, G, nc;
};

// dt_raw of token row t for head h (0 past the sequence's end); loaded a
// head ahead of its use so that its latency hides behind the head before
__device__ inline float row_dt_raw(const TcParams& p, int bi, int h, int t, bool valid)
{
    return valid ? __bfloat162float(p.dt_raw[((size_t)bi * p.L + t) * p.H + h]) : 0.0f;
}

// dt_t and sigmoid(dt_raw + dt_bias) from the raw value (dt = 0 past the end)
__device__ inline void row_dt(float bias, float raw, bool valid, float& dt, float& sig)
{
    const float v = valid ? raw + bias : 0.0f;
    dt = valid ? softplus_f(v) : 0.0f;
    sig = 1.0f / (1.0f + __expf(-v));
}

// Inclusive cumsum of l over the 128 rows held by 4 warps (one row per
// thread, warp w%4 = quadrant): warp scans, then the lower quadrants' totals.
// `tot` is 4 floats of shared memory; `bar_id` a named barrier of the 128 threads.
__device__ inline float block_cumsum128(float l, int quad, int lane, float* tot, int bar_id)
{
    const float inc = warp_incl_scan(l, lane);
    if (lane == 31) tot[quad] = inc;
    named_bar_sync(bar_id, 128);
    float off = 0.0f;
    for (int q = 0; q < quad; ++q) off += tot[q];
    return inc + off;
}

// ---------------------------------------------------------------------------
// Kernel 1: chunk states S^T = B^T (w o X) and dS^T = C^T (Ec o dY)
// ---------------------------------------------------------------------------
namespace k1 {
constexpr int kEwWarps = 8;                     // two per TMEM lane quadrant
constexpr int kThreads = (kEwWarps + 2) * 32;   // warp 0 producer, 1 MMA, 2..9 rows
// X and dY are scaled in place (w o X, Ec o dY); 2 CTAs fit on an SM
constexpr int kOffB = 0, kOffC = 32768, kOffX = 65536, kOffDY = 81920;
constexpr int kOffVec = 98304;                  // floats: tot[4], w[128], Ec[128], A and dt_bias [kMaxHpg]
constexpr int kOffBar = kOffVec + 1088 + 8 * kMaxHpg;
constexpr int kOffMisc = kOffBar + 8 * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr uint32_t kTmemCols = 128;             // S^T [0,64), dS^T [64,128)
constexpr uint32_t kIdS = umma_idesc_bf16(128, 64, true, true);   // B^T (MN) x wX (MN)
}  // namespace k1

__global__ void __launch_bounds__(k1::kThreads, 2)
bwd_states_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmDY,
                  const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmdS,
                  const TcParams p)
{
    using namespace k1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const int bi = blockIdx.y / p.G, g = blockIdx.y - bi * p.G;
    const int hpg = p.H / p.G;
    const int t0 = c * kQ;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* bar_ld = bars + 0;     // X, dY (and B, C for the first head) landed
    uint64_t* bar_w = bars + 1;      // w o X and Ec o dY written in place (row warps)
    uint64_t* bar_mma = bars + 2;    // S^T, dS^T in TMEM (X and dY free)
    uint64_t* bar_staged = bars + 3; // S^T, dS^T staged in bf16 over X and dY (row warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* aborted = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    float* tot = reinterpret_cast<float*>(smem + kOffVec);
    float* sA = tot + 4 + 2 * kQ;      // [hpg] A of the group's heads
    float* sBias = sA + kMaxHpg;       // [hpg] dt_bias
    for (int k = tid; k < hpg; k += kThreads) {
        sA[k] = p.A[g * hpg + k];
        sBias[k] = p.dt_bias ? p.dt_bias[g * hpg + k] : 0.0f;
    }

    if (tid == 0) {
        *aborted = 0;
        mbar_init(bar_ld, 1);
        mbar_init(bar_w, kEwWarps * 32);
        mbar_init(bar_mma, 1);
        mbar_init(bar_staged, kEwWarps * 32);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmC);
            prefetch_tensormap(&tmDY);
            prefetch_tensormap(&tmS);
            prefetch_tensormap(&tmdS);
            // the staged S^T and dS^T tiles of head hh go out by TMA store;
            // X and dY are reloaded once the store has read them
            auto store_states = [&](int hh) {
                const int row = ((bi * p.H + g * hpg + hh) * p.nc + c) * kN;
                tma_store_3d(&tmS, smem + kOffX, 0, row, 0);
                tma_store_3d(&tmdS, smem + kOffDY, 0, row, 0);
                bulk_commit_group();
                bulk_wait_group_read0();
            };
            int issued = 0;
            for (int hh = 0; hh < hpg; ++hh) {
                const int h = g * hpg + hh;
                if (hh > 0) {
                    if (!mbar_wait_bounded(bar_staged, (uint32_t)(hh - 1) & 1u, kWaitNs, aborted, p.status)) break;
                    store_states(hh - 1);
                }
                mbar_arrive_expect_tx(bar_ld, hh == 0 ? 6 * kTileHalf : 2 * kTileHalf);
                tma_load_3d(smem + kOffX, &tmX, h * kP, t0, bi, bar_ld);
                tma_load_3d(smem + kOffDY, &tmDY, h * kP, t0, bi, bar_ld);
                if (hh == 0) {
                    tma_load_3d(smem + kOffB, &tmB, g * kN, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffB + kTileHalf, &tmB, g * kN + 64, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffC, &tmC, g * kN, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffC + kTileHalf, &tmC, g * kN + 64, t0, bi, bar_ld);
                }
                if (hh + 1 < hpg) {   // the next head's tiles into L2 meanwhile
                    tma_prefetch_l2_3d(&tmX, (h + 1) * kP, t0, bi);
                    tma_prefetch_l2_3d(&tmDY, (h + 1) * kP, t0, bi);
                }
                ++issued;
            }
            if (issued == hpg && mbar_wait_bounded(bar_staged, (uint32_t)(hpg - 1) & 1u, kWaitNs, aborted, p.status))
                store_states(hpg - 1);
            if (issued > 0) drain_wait(bar_ld, (uint32_t)(issued - 1) & 1u);
            bulk_wait_group0();
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t sB = smem_u32(smem + kOffB), sC = smem_u32(smem + kOffC);
            const uint32_t sWX = smem_u32(smem + kOffX), sWDY = smem_u32(smem + kOffDY);   // scaled in place
            int committed = 0;
            for (int hh = 0; hh < hpg; ++hh) {
                const uint32_t ph = (uint32_t)hh & 1u;
                // (the row warps waited for the loads before arriving here; a
                // second waiter on bar_ld could fall two phases behind it)
                if (!mbar_wait_bounded(bar_w, ph, kWaitNs, aborted, p.status)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_bf16(tmem, desc_mn(sB, k), desc_mn(sWX, k), kIdS, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_bf16(tmem + 64, desc_mn(sC, k), desc_mn(sWDY, k), kIdS, k > 0);
                umma_commit(bar_mma);
                ++committed;
            }
            if (committed > 0) drain_wait(bar_mma, (uint32_t)(committed - 1) & 1u);
        }
        __syncwarp();
    } else {
        // elementwise warps, two per lane quadrant (part 0, 1): thread = token
        // row i (weights; part p scales chunks 4p..4p+3 of X and dY), then
        // state row n = i (epilogue: part 0 writes S^T, part 1 dS^T)
        const int ew = warp - 2;
        const int quad = warp & 3;
        const int part = ew >> 2;
        const int i = quad * 32 + lane;
        const int t = t0 + i;
        const bool valid = t < p.L;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float* sW = tot + 4;   // [128] w_i = El_i dt_i
        float* sE = sW + kQ;   // [128] Ec_i
        bool ok = true;
        float raw_next = part == 0 ? row_dt_raw(p, bi, g * hpg, t, valid) : 0.0f;
        for (int hh = 0; hh < hpg; ++hh) {
            const int h = g * hpg + hh;
            const int chain = bi * p.H + h;
            const uint32_t ph = (uint32_t)hh & 1u;
            const float raw = raw_next;
            if (part == 0 && hh + 1 < hpg) raw_next = row_dt_raw(p, bi, h + 1, t, valid);
            // the previous head's weights read; a give-up anywhere ends all rows here
            if (named_bar_any(2, kEwWarps * 32, !ok)) break;
            if (part == 0) {
                float dt, sig;
                row_dt(sBias[hh], raw, valid, dt, sig);
                const float cum = block_cumsum128(dt * sA[hh] * kLog2e, quad, lane, tot, 1);
                const float cl = tot[0] + tot[1] + tot[2] + tot[3];
                sW[i] = ex2_approx(cl - cum) * dt;
                sE[i] = ex2_approx(cum);
                if (i == 0) p.ws_cl[(size_t)chain * p.nc + c] = cl;
            }
            named_bar_sync(2, kEwWarps * 32);
            const float w = sW[i], e = sE[i];
            // (after a give-up the head runs on without waiting, so that
            // every row reaches the next barrier)
            ok = mbar_wait_bounded(bar_ld, ph, kWaitNs, aborted, p.status) && ok;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float v[8];
                const uint32_t o = sw128(i, part * 4 + cc);
                unpack8(*reinterpret_cast<const uint4*>(smem + kOffX + o), v);
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] *= w;
                *reinterpret_cast<uint4*>(smem + kOffX + o) = pack8(v);
                unpack8(*reinterpret_cast<const uint4*>(smem + kOffDY + o), v);
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] *= e;
                *reinterpret_cast<uint4*>(smem + kOffDY + o) = pack8(v);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_w);
            ok = mbar_wait_bounded(bar_mma, ph, kWaitNs, aborted, p.status) && ok;
            tc_fence_after_sync();
            // state row n = i of S^T (part 0) or dS^T (part 1), in bf16, staged
            // (swizzled as the store's tensor map expects) over X or dY
            uint8_t* stg = smem + (part == 0 ? kOffX : kOffDY);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(part * 64 + half * 32), v);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(stg + sw128(i, half * 4 + k)) = pack8(v + 8 * k);
            }
            tc_fence_before_sync();
            fence_proxy_async_smem();
            mbar_arrive(bar_staged);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: entering states forward, state gradients backward
// ---------------------------------------------------------------------------
// Grid (chains, kPassSlices, 2): thread j of slice s owns state elements
// e = s*1024 + 4j .. +3 of the [n][p] layout (one n, four p); z = 0 walks
// the entering states forward, z = 1 the state gradients backward.
__device__ inline void st_bf16x4(__nv_bfloat16* dst, const float (&v)[4])
{
    __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
}

__global__ void __launch_bounds__(kPassThreads)
bwd_pass_kernel(const TcParams p)
{
    const int chain = blockIdx.x, s = blockIdx.y;
    const bool fwd = blockIdx.z == 0;
    const int e0 = s * (kStatesDim / kPassSlices) + threadIdx.x * 4;
    const int n = e0 / kP, p0 = e0 - n * kP;
    const int nc = p.nc;
    const size_t base = (size_t)chain * nc * kStatesDim + e0;
    const float* cl = p.ws_cl + (size_t)chain * nc;
    const float* start = fwd ? p.init_state : p.dfinal;
    const __nv_bfloat16* inc = fwd ? p.ws_S : p.ws_dS;
    __nv_bfloat16* out = fwd ? p.ws_hb : p.ws_gb;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = start ? start[(size_t)chain * kStatesDim + (size_t)(p0 + k) * kN + n] : 0.0f;
    // forward: out[c] = h0_c, h0_{c+1} = 2^cl_c h0_c + S_c;
    // backward: out[c] = g_c, g_{c-1} = 2^cl_c g_c + dS_c.
    // The chunk states and decays are loaded kAhead chunks ahead (a ring
    // of registers with static indices), so the walk is not one load
    // latency per chunk.
    constexpr int kAhead = 4;
    uint2 ring[kAhead];
    float dring[kAhead];
    auto chunk_of = [&](int k) { return fwd ? k : nc - 1 - k; };
#pragma unroll
    for (int r = 0; r < kAhead; ++r) {
        if (r < nc) {
            const int c = chunk_of(r);
            ring[r] = *reinterpret_cast<const uint2*>(inc + base + (size_t)c * kStatesDim);
            dring[r] = cl[c];
        }
    }
    for (int k0 = 0; k0 < nc; k0 += kAhead) {
#pragma unroll
        for (int r = 0; r < kAhead; ++r) {
            const int k = k0 + r;
            if (k < nc) {
                const int c = chunk_of(k);
                const uint2 q = ring[r];
                const float d = ex2_approx(dring[r]);
                if (k + kAhead < nc) {
                    const int cn = chunk_of(k + kAhead);
                    ring[r] = *reinterpret_cast<const uint2*>(inc + base + (size_t)cn * kStatesDim);
                    dring[r] = cl[cn];
                }
                st_bf16x4(out + base + (size_t)c * kStatesDim, v);
                const float a[4] = {__uint_as_float(q.x << 16), __uint_as_float(q.x & 0xffff0000u),
                                    __uint_as_float(q.y << 16), __uint_as_float(q.y & 0xffff0000u)};
#pragma unroll
                for (int e = 0; e < 4; ++e) v[e] = fmaf(d, v[e], a[e]);
            }
        }
    }
    if (!fwd && p.dinit) {
#pragma unroll
        for (int k = 0; k < 4; ++k) p.dinit[(size_t)chain * kStatesDim + (size_t)(p0 + k) * kN + n] = v[k];
    }
}

// ---------------------------------------------------------------------------
// Kernel 3: the chunk's gradients
// ---------------------------------------------------------------------------
namespace k3 {
constexpr int kEwWarps = 16;                    // 4 lane quadrants x 4 column quarters
constexpr int kEwThreads = kEwWarps * 32;
constexpr int kThreads = kEwThreads + 64;       // warp 0 producer, 1 MMA, 2..17 elementwise
// shared memory (1024-aligned); region R holds X, h0, Ec o dY, dt o El o X
// in the first phase and the tiles M1, M3 in the second
constexpr int kOffB = 0, kOffC = 32768, kOffDY = 65536, kOffG = 81920, kOffR = 98304;
constexpr int kOffX = kOffR, kOffH = kOffR + 16384, kOffEDY = kOffR + 32768, kOffEX = kOffR + 49152;
constexpr int kOffM1 = kOffR, kOffM3 = kOffR + 32768;
// floats, two sets by head parity: cum, dt, sig, v [128] each, partials
// [6][4][128], t1 [16]; then scan scratch [16]; A, D, dt_bias [kMaxHpg]
constexpr int kOffVec = kOffR + 65536;
constexpr int kVecSet = 4 * kQ + 24 * kQ + 16;
constexpr int kVecFloats = 2 * kVecSet + 16 + 3 * kMaxHpg;
constexpr int kOffBar = kOffVec + ((kVecFloats * 4 + 63) / 64) * 64;
constexpr int kNumBars = 7;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr uint32_t kTmemCols = 512;
// TMEM columns
constexpr uint32_t kColYX = 0;     // YX [0,128); after the tiles are built: gB [0,64), B g^T [64,128)
constexpr uint32_t kColGB = 0, kColBG = 64;
constexpr uint32_t kColCB = 128;   // CB (kept across the group's heads)
constexpr uint32_t kColDC = 256;   // dC, summed over the group's heads
constexpr uint32_t kColDB = 384;   // dB, summed over the group's heads
constexpr uint32_t kIdKK128 = umma_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdKM128 = umma_idesc_bf16(128, 128, false, true);
constexpr uint32_t kIdMM128 = umma_idesc_bf16(128, 128, true, true);
constexpr uint32_t kIdMM64 = umma_idesc_bf16(128, 64, true, true);
constexpr uint32_t kIdKM64 = umma_idesc_bf16(128, 64, false, true);
constexpr int kBarEw = 1, kBarRows = 2;         // named barriers: all elementwise warps; the 4 row warps
}  // namespace k3

__global__ void __launch_bounds__(k3::kThreads, 1)
bwd_chunk_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmDY,
                 const __grid_constant__ CUtensorMap tmHb, const __grid_constant__ CUtensorMap tmGb, const TcParams p)
{
    using namespace k3;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const int bi = blockIdx.y / p.G, g = blockIdx.y - bi * p.G;
    const int hpg = p.H / p.G;
    const int t0 = c * kQ;
    const int q = min(kQ, p.L - t0);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* bar_ld = bars + 0;   // X, dY, h0, g (and B, C for the first head) landed
    uint64_t* bar_e0 = bars + 1;   // Ec o dY, dt o El o X written
    uint64_t* bar_p1 = bars + 2;   // YX, CB and the first products of dC, dB done
    uint64_t* bar_e1 = bars + 3;   // M1, M3 written; YX read
    uint64_t* bar_p2 = bars + 4;   // dC, dB, gB, B g^T done
    uint64_t* bar_e2 = bars + 5;   // the head's epilogue has read gB, B g^T and dC
    uint64_t* bar_p2a = bars + 6;  // gB, B g^T done (the rest of the second products still running)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* aborted = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    // per-head vectors and partial sums, by head parity (a head's last step
    // runs while the next head is under way)
    struct Vec {
        float *cum, *dt, *sig;
        float* v;                                    // 2^(cum_e - cum_j), e = last column of j's 32-block
        float *row, *rowd, *dd, *dcc, *xgb, *col;   // [4][128] partials
        float* t1;                                   // [16] <g, h0> partials
    };
    auto vec = [&](int parity) {
        float* b = reinterpret_cast<float*>(smem + kOffVec) + parity * kVecSet;
        Vec v;
        v.cum = b;
        v.dt = b + kQ;
        v.sig = b + 2 * kQ;
        v.v = b + 3 * kQ;
        v.row = b + 4 * kQ;       // [column quarter][row]: W partials
        v.rowd = v.row + 4 * kQ;  // rowD partials
        v.dd = v.rowd + 4 * kQ;   // dy.x partials
        v.dcc = v.dd + 4 * kQ;    // dC.C partials
        v.xgb = v.dcc + 4 * kQ;   // x^T g B partials
        v.col = v.xgb + 4 * kQ;   // [lane quadrant][column]: sum_k M2 CB partials
        v.t1 = v.col + 4 * kQ;
        return v;
    };
    float* tot = reinterpret_cast<float*>(smem + kOffVec) + 2 * kVecSet;   // [4] cumsum, [8] row scans
    float* sA = tot + 16;              // [hpg] per-head scalars of the group
    float* sD = sA + kMaxHpg;
    float* sBias = sD + kMaxHpg;
    for (int k = tid; k < hpg; k += kThreads) {
        sA[k] = p.A[g * hpg + k];
        sD[k] = p.D ? p.D[g * hpg + k] : 0.0f;
        sBias[k] = p.dt_bias ? p.dt_bias[g * hpg + k] : 0.0f;
    }

    if (tid == 0) {
        *aborted = 0;
        mbar_init(bar_ld, 1);
        mbar_init(bar_e0, kEwThreads);
        mbar_init(bar_p1, 1);
        mbar_init(bar_e1, kEwThreads);
        mbar_init(bar_p2, 1);
        mbar_init(bar_e2, kEwThreads);
        mbar_init(bar_p2a, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmC);
            prefetch_tensormap(&tmDY);
            prefetch_tensormap(&tmHb);
            prefetch_tensormap(&tmGb);
            int issued = 0;
            for (int hh = 0; hh < hpg; ++hh) {
                const int h = g * hpg + hh;
                const int row = ((bi * p.H + h) * p.nc + c) * kN;   // state rows of this (chain, chunk)
                // the previous head's products are done: X, h0, dY, g and the
                // M tiles are free (its epilogue reads x and dy from global memory)
                if (hh > 0 && !mbar_wait_bounded(bar_p2, (uint32_t)(hh - 1) & 1u, kWaitNs, aborted, p.status))
                    break;
                mbar_arrive_expect_tx(bar_ld, hh == 0 ? 8 * kTileHalf : 4 * kTileHalf);
                tma_load_3d(smem + kOffX, &tmX, h * kP, t0, bi, bar_ld);
                tma_load_3d(smem + kOffDY, &tmDY, h * kP, t0, bi, bar_ld);
                tma_load_3d(smem + kOffH, &tmHb, 0, row, 0, bar_ld);
                tma_load_3d(smem + kOffG, &tmGb, 0, row, 0, bar_ld);
                if (hh == 0) {
                    tma_load_3d(smem + kOffB, &tmB, g * kN, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffB + kTileHalf, &tmB, g * kN + 64, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffC, &tmC, g * kN, t0, bi, bar_ld);
                    tma_load_3d(smem + kOffC + kTileHalf, &tmC, g * kN + 64, t0, bi, bar_ld);
                }
                if (hh + 1 < hpg) {   // the next head's tiles into L2 while this head computes
                    tma_prefetch_l2_3d(&tmX, (h + 1) * kP, t0, bi);
                    tma_prefetch_l2_3d(&tmDY, (h + 1) * kP, t0, bi);
                    tma_prefetch_l2_3d(&tmHb, 0, row + p.nc * kN, 0);
                    tma_prefetch_l2_3d(&tmGb, 0, row + p.nc * kN, 0);
                }
                ++issued;
            }
            if (issued > 0) drain_wait(bar_ld, (uint32_t)(issued - 1) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
            const uint32_t sB = smem_u32(smem + kOffB), sC = smem_u32(smem + kOffC);
            const uint32_t sDY = smem_u32(smem + kOffDY), sG = smem_u32(smem + kOffG);
            const uint32_t sX = smem_u32(smem + kOffX), sH = smem_u32(smem + kOffH);
            const uint32_t sEDY = smem_u32(smem + kOffEDY), sEX = smem_u32(smem + kOffEX);
            const uint32_t sM1 = smem_u32(smem + kOffM1), sM3 = smem_u32(smem + kOffM3);
            int committed = 0;
            for (int hh = 0; hh < hpg; ++hh) {
                const uint32_t ph = (uint32_t)hh & 1u;
                const uint32_t acc = hh > 0 ? 1u : 0u;   // dC, dB: sums over the group's heads
                if (!mbar_wait_bounded(bar_ld, ph, kWaitNs, aborted, p.status)) break;
                // the previous head's epilogue has read gB, B g^T (YX's columns) and dC
                if (hh > 0 && !mbar_wait_bounded(bar_e2, ph ^ 1u, kWaitNs, aborted, p.status)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 4; ++k)   // YX = dY X^T (K = P)
                    umma_bf16(tmem + kColYX, desc_k(sDY, k), desc_k(sX, k), kIdKK128, k > 0);
                if (hh == 0) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)   // CB = C B^T (K = N)
                        umma_bf16(tmem + kColCB, desc_k(sC, k), desc_k(sB, k), kIdKK128, k > 0);
                }
                if (!mbar_wait_bounded(bar_e0, ph, kWaitNs, aborted, p.status)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 4; ++k)   // dC (+)= (Ec o dY) h0      (h0 as [n][p], K = P)
                    umma_bf16(tmem + kColDC, desc_k(sEDY, k), desc_k(sH, k), kIdKK128, k > 0 ? 1u : acc);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // dB (+)= (dt o El o X) g
                    umma_bf16(tmem + kColDB, desc_k(sEX, k), desc_k(sG, k), kIdKK128, k > 0 ? 1u : acc);
                umma_commit(bar_p1);
                ++committed;
                if (!mbar_wait_bounded(bar_e1, ph, kWaitNs, aborted, p.status)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)   // gB = M3^T dY
                    umma_bf16(tmem + kColGB, desc_mn(sM3, k), desc_mn(sDY, k), kIdMM64, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)   // B g^T                       (g as [n][p], K = N)
                    umma_bf16(tmem + kColBG, desc_k(sB, k), desc_mn(sG, k), kIdKM64, k > 0);
                umma_commit(bar_p2a);         // dx can start
#pragma unroll
                for (int k = 0; k < 8; ++k)   // dC += M1 B                 (K = Q)
                    umma_bf16(tmem + kColDC, desc_k(sM1, k), desc_mn(sB, k), kIdKM128, 1u);
#pragma unroll
                for (int k = 0; k < 8; ++k)   // dB += M1^T C  (M1 = dt_j o M2)
                    umma_bf16(tmem + kColDB, desc_mn(sM1, k), desc_mn(sC, k), kIdMM128, 1u);
                umma_commit(bar_p2);
                ++committed;
            }
            if (committed > 0) drain_wait((committed & 1) ? bar_p1 : bar_p2, (uint32_t)((committed - 1) >> 1) & 1u);
        }
        __syncwarp();
    } else {
        // ---------------- elementwise warps ----------------
        const int ew = warp - 2;
        const int quad = warp & 3;           // TMEM lane quadrant: rows 32*quad ..
        const int qs = ew >> 2;              // column quarter
        const int i = quad * 32 + lane;      // token row
        const int t = t0 + i;
        const bool valid = i < q;
        const size_t trow = (size_t)bi * p.L + min(t, p.L - 1);   // (a valid row for addressing)
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        // dC and dB accumulate over the group's heads in TMEM; a head's dC.C
        // is the difference of consecutive running dots
        float prev_dcc = 0.0f;
        bool ok = true;
        float raw_next = qs == 0 ? row_dt_raw(p, bi, g * hpg, t, valid) : 0.0f;

        // The last step of head hh, on the row warps (qs == 0): per-token
        // scalars, the decay gradient, ddt_raw and the partial sums of dA,
        // dD, ddt_bias.  It runs one head late, while the next head's second
        // products are on the tensor cores.
        auto row_step = [&](int hh) {
            const Vec v = vec(hh & 1);
            const int h = g * hpg + hh;
            const int chain = bi * p.H + h;
            const float cl = v.cum[kQ - 1];
            const float dt_i = v.dt[i];
            const float El = ex2_approx(cl - v.cum[i]);
            const float dcc_h = v.dcc[i] + v.dcc[kQ + i] + v.dcc[2 * kQ + i] + v.dcc[3 * kQ + i];
            const float xgb = v.xgb[i] + v.xgb[kQ + i] + v.xgb[2 * kQ + i] + v.xgb[3 * kQ + i];
            const float col = v.col[i] + v.col[kQ + i] + v.col[2 * kQ + i] + v.col[3 * kQ + i];
            const float wr = v.row[i] + v.row[kQ + i] + v.row[2 * kQ + i] + v.row[3 * kQ + i];
            const float rowd = v.rowd[i] + v.rowd[kQ + i] + v.rowd[2 * kQ + i] + v.rowd[3 * kQ + i];
            const float dd = v.dd[i] + v.dd[kQ + i] + v.dd[2 * kQ + i] + v.dd[3 * kQ + i];
            const float ub = fmaf(El, xgb, col);   // U_i . B_i
            const float a = dt_i * ub;
            const float dcc = dcc_h - rowd;        // dC.C with M1's rounding taken out
            // exclusive prefix of a, inclusive suffix of dcc, total of wr
            const float ia = warp_incl_scan(a, lane);
            const float idc = warp_incl_scan(dcc, lane);
            const float tw = warp_total(wr);
            float* ts = tot + 4;
            named_bar_sync(kBarRows, 128);   // ts[] of the previous step read
            if (lane == 31) {
                ts[quad] = ia;
                ts[4 + quad] = idc;
            }
            named_bar_sync(kBarRows, 128);
            float offa = 0.0f, offc = 0.0f, alldc = 0.0f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                if (qq < quad) {
                    offa += ts[qq];
                    offc += ts[4 + qq];
                }
                alldc += ts[4 + qq];
            }
            named_bar_sync(kBarRows, 128);
            if (lane == 0) ts[quad] = tw;
            named_bar_sync(kBarRows, 128);
            const float wsum = ts[0] + ts[1] + ts[2] + ts[3];
            float t1 = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < kEwWarps; ++w2) t1 += v.t1[w2];
            t1 *= ex2_approx(cl);
            const float pre = offa + ia - a;                  // sum_{j<i} a_j
            const float suf = alldc - (offc + idc - dcc);     // sum_{k>=i} dcc_k
            const float r = t1 - wsum + pre + suf;
            float ra = 0.0f, rd = 0.0f, rb = 0.0f;
            if (valid) {
                const float ddt = ub + sA[hh] * r;
                const float dv = ddt * v.sig[i];
                p.ddt_raw[trow * p.H + h] = __float2bfloat16_rn(dv);
                ra = dt_i * r;
                rd = dd;
                rb = dv;
            }
            ra = warp_total(ra);
            rd = warp_total(rd);
            rb = warp_total(rb);
            if (lane == 0) {
                const size_t nparts = (size_t)p.b * p.H * p.nc * kParts;
                const size_t o = ((size_t)chain * p.nc + c) * kParts + quad;
                p.ws_part[o] = ra;
                p.ws_part[nparts + o] = rd;
                p.ws_part[2 * nparts + o] = rb;
            }
        };

        for (int hh = 0; hh < hpg; ++hh) {
            const int h = g * hpg + hh;
            const uint32_t ph = (uint32_t)hh & 1u;
            const Vec v = vec(hh & 1);
            const float Ah = sA[hh];
            const float Dh = sD[hh];
            const float raw = raw_next;
            if (qs == 0 && hh + 1 < hpg) raw_next = row_dt_raw(p, bi, h + 1, t, valid);

            // E0: dt, cumulative decay (row warps), then the scaled copies.
            // The barrier also ends the loop of every warp at once after a
            // give-up (inside a head nobody leaves early, so that every
            // warp reaches every barrier), and it orders the previous
            // head's partial sums before their use.
            if (named_bar_any(kBarEw, kEwThreads, !ok)) {
                ok = false;
                break;
            }
            if (qs == 0) {
                float dt, sig;
                row_dt(sBias[hh], raw, valid, dt, sig);
                const float cum = block_cumsum128(dt * Ah * kLog2e, quad, lane, tot, kBarRows);
                v.cum[i] = cum;
                v.dt[i] = dt;
                v.sig[i] = sig;
                // (this warp holds the 32-block of row i: its last row is lane 31)
                v.v[i] = ex2_approx(__shfl_sync(0xffffffffu, cum, 31) - cum);
            }
            named_bar_sync(kBarEw, kEwThreads);
            const float cum_i = v.cum[i], dt_i = v.dt[i];
            const float cl = v.cum[kQ - 1];
            const float Ec = ex2_approx(cum_i), El = ex2_approx(cl - cum_i);
            ok = mbar_wait_bounded(bar_ld, ph, kWaitNs, aborted, p.status) && ok;
            {
                float dd = 0.0f;
                const float wx = dt_i * El;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t o = sw128(i, qs * 2 + cc);
                    float y[8], xv[8];
                    unpack8(*reinterpret_cast<const uint4*>(smem + kOffDY + o), y);
                    unpack8(*reinterpret_cast<const uint4*>(smem + kOffX + o), xv);
#pragma unroll
                    for (int k = 0; k < 8; ++k) dd = fmaf(y[k], xv[k], dd);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        y[k] *= Ec;
                        xv[k] *= wx;
                    }
                    *reinterpret_cast<uint4*>(smem + kOffEDY + o) = pack8(y);
                    *reinterpret_cast<uint4*>(smem + kOffEX + o) = pack8(xv);
                }
                v.dd[qs * kQ + i] = dd;
                // <g, h0> over the two bf16 tiles (same layout): 2 chunks per thread
                float gh = 0.0f;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t o = (uint32_t)((ew * 32 + lane) * 2 + cc) * 16u;
                    float hv[8], gv[8];
                    unpack8(*reinterpret_cast<const uint4*>(smem + kOffH + o), hv);
                    unpack8(*reinterpret_cast<const uint4*>(smem + kOffG + o), gv);
#pragma unroll
                    for (int k = 0; k < 8; ++k) gh = fmaf(hv[k], gv[k], gh);
                }
                gh = warp_total(gh);
                if (lane == 0) v.t1[ew] = gh;
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_e0);

            // E1: the masked tiles M1, M3 from YX and CB; W's row partials,
            // the rounding of M1 (rowD) and the column sums of M2 o CB
            ok = mbar_wait_bounded(bar_p1, ph, kWaitNs, aborted, p.status) && ok;
            tc_fence_after_sync();
            {
                // Column block qs against the row block quad: above the
                // diagonal the tiles are zero; below it the decay factors
                // as 2^(cum_i - cum_e) 2^(cum_e - cum_j) (e = the block's
                // last column, both factors <= 1); on the diagonal one
                // exponential per element.
                float w = 0.0f, rowd = 0.0f;
                const uint32_t half = (uint32_t)(qs >> 1) * kTileHalf;
                const bool above = qs > quad, below = qs < quad;
                const float u = below ? ex2_approx(cum_i - v.cum[qs * 32 + 31]) : 0.0f;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {   // 16 columns at a time
                    float cs = 0.0f;
                    if (above) {
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const uint32_t o = half + sw128(i, (qs & 1) * 4 + sub * 2 + cc);
                            *reinterpret_cast<uint4*>(smem + kOffM1 + o) = z;
                            *reinterpret_cast<uint4*>(smem + kOffM3 + o) = z;
                        }
                    } else {
                        float yx[16], cb[16], col[16];
                        tmem_ld16(tmem + kColYX + lane_off + (uint32_t)(qs * 32 + sub * 16), yx);
                        tmem_ld16(tmem + kColCB + lane_off + (uint32_t)(qs * 32 + sub * 16), cb);
                        tmem_wait_ld();
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int j0 = qs * 32 + sub * 16 + cc * 8;
                            float lm[8];
                            if (below) {
                                const float4 va = reinterpret_cast<const float4*>(v.v + j0)[0];
                                const float4 vb = reinterpret_cast<const float4*>(v.v + j0)[1];
                                const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                                for (int k = 0; k < 8; ++k) lm[k] = u * vv[k];
                            } else {
                                const float4 ca = reinterpret_cast<const float4*>(v.cum + j0)[0];
                                const float4 cb4 = reinterpret_cast<const float4*>(v.cum + j0)[1];
                                const float cj[8] = {ca.x, ca.y, ca.z, ca.w, cb4.x, cb4.y, cb4.z, cb4.w};
#pragma unroll
                                for (int k = 0; k < 8; ++k) lm[k] = j0 + k <= i ? ex2_approx(cum_i - cj[k]) : 0.0f;
                            }
                            const float4 da = reinterpret_cast<const float4*>(v.dt + j0)[0];
                            const float4 db = reinterpret_cast<const float4*>(v.dt + j0)[1];
                            const float dj[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
                            float m1[8], m3[8];
#pragma unroll
                            for (int k = 0; k < 8; k += 2) {
                                const int jj = cc * 8 + k;
                                const float2 v2 = mul2(make_float2(lm[k], lm[k + 1]), make_float2(yx[jj], yx[jj + 1]));
                                const float2 v1 = mul2(v2, make_float2(dj[k], dj[k + 1]));
                                const float2 c2 = make_float2(cb[jj], cb[jj + 1]);
                                m1[k] = bf16_round(v1.x);
                                m1[k + 1] = bf16_round(v1.y);
                                const float2 m3p = mul2(make_float2(lm[k], lm[k + 1]), c2);
                                m3[k] = m3p.x;
                                m3[k + 1] = m3p.y;
                                w = fmaf(v1.x, c2.x, fmaf(v1.y, c2.y, w));
                                rowd = fmaf(m1[k] - v1.x, c2.x, fmaf(m1[k + 1] - v1.y, c2.y, rowd));
                                const float2 cl2 = mul2(v2, c2);
                                col[jj] = cl2.x;
                                col[jj + 1] = cl2.y;
                            }
                            const uint32_t o = half + sw128(i, (qs & 1) * 4 + sub * 2 + cc);
                            *reinterpret_cast<uint4*>(smem + kOffM1 + o) = pack8(m1);
                            *reinterpret_cast<uint4*>(smem + kOffM3 + o) = pack8(m3);
                        }
                        cs = warp_colsum16(col, lane);
                    }
                    if (lane < 16) v.col[quad * kQ + qs * 32 + sub * 16 + lane] = cs;
                }
                v.row[qs * kQ + i] = w;
                v.rowd[qs * kQ + i] = rowd;
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_e1);

            // the previous head's last step, while the products run
            if (qs == 0 && hh > 0) row_step(hh - 1);

            // E2: dx, this head's dC.C and x^T g B partials (the dy and x
            // rows are loaded before the wait for the products)
            const size_t rowp = (trow * p.H + h) * kP + qs * 16;
            const uint4* dyr = reinterpret_cast<const uint4*>(p.dy + rowp);
            const uint4* xr = reinterpret_cast<const uint4*>(p.x + trow * p.row_stride + (size_t)h * kP + qs * 16);
            const uint4 dy0 = dyr[0], dy1 = dyr[1], x0 = xr[0], x1 = xr[1];
            ok = mbar_wait_bounded(bar_p2a, ph, kWaitNs, aborted, p.status) && ok;
            tc_fence_after_sync();
            {
                // dx and x^T g B from gB and B g^T, while dC and dB are still
                // on the tensor cores
                float gb[16], bg[16];
                tmem_ld16(tmem + kColGB + lane_off + (uint32_t)(qs * 16), gb);
                tmem_ld16(tmem + kColBG + lane_off + (uint32_t)(qs * 16), bg);
                tmem_wait_ld();
                float dxv[16], xgb = 0.0f;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float y[8], xv[8];
                    unpack8(cc ? dy1 : dy0, y);
                    unpack8(cc ? x1 : x0, xv);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        dxv[cc * 8 + k] = fmaf(Dh, y[k], dt_i * fmaf(El, bg[cc * 8 + k], gb[cc * 8 + k]));
                        xgb = fmaf(xv[k], bg[cc * 8 + k], xgb);
                    }
                }
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(p.dx + rowp);
                    dst[0] = pack8(dxv);
                    dst[1] = pack8(dxv + 8);
                }
                v.xgb[qs * kQ + i] = xgb;
            }
            ok = mbar_wait_bounded(bar_p2, ph, kWaitNs, aborted, p.status) && ok;
            tc_fence_after_sync();
            {
                // this head's dC.C: the difference of consecutive running dots
                const uint32_t half = (uint32_t)(qs >> 1) * kTileHalf;
                float vv[32];
                tmem_ld32(tmem + kColDC + lane_off + (uint32_t)(qs * 32), vv);
                tmem_wait_ld();
                float dcc = 0.0f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float cr[8];
                    unpack8(*reinterpret_cast<const uint4*>(smem + kOffC + half + sw128(i, (qs & 1) * 4 + cc)), cr);
#pragma unroll
                    for (int k = 0; k < 8; ++k) dcc = fmaf(vv[cc * 8 + k], cr[k], dcc);
                }
                const float run = dcc;
                v.dcc[qs * kQ + i] = run - prev_dcc;
                prev_dcc = run;
            }
            tc_fence_before_sync();
            mbar_arrive(bar_e2);   // gB, B g^T and dC read: the next head's products may start
        }
        // the last head's last step (its partial sums complete after this
        // barrier, which also makes the decision the same for every warp)
        if (named_bar_any(kBarEw, kEwThreads, !ok)) ok = false;
        if (ok && qs == 0) row_step(hpg - 1);
        // dB, dC of the group: this thread's row and 32 columns (the last
        // head's products are complete: its epilogue waited for them)
        if (ok) {
            tc_fence_after_sync();
            float vc[32], vb[32];
            tmem_ld32(tmem + kColDC + lane_off + (uint32_t)(qs * 32), vc);
            tmem_ld32(tmem + kColDB + lane_off + (uint32_t)(qs * 32), vb);
            tmem_wait_ld();
            if (valid) {
                const size_t o = ((trow * p.G) + g) * kN + qs * 32;
                uint4* db = reinterpret_cast<uint4*>(p.dB + o);
                uint4* dc = reinterpret_cast<uint4*>(p.dC + o);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    db[cc] = pack8(vb + cc * 8);
                    dc[cc] = pack8(vc + cc * 8);
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// dA, dD, ddt_bias [H]: one CTA per head sums its (sequence, chunk, quarter)
// partials in a fixed order (thread-strided, then a fixed tree).
__global__ void __launch_bounds__(256)
bwd_head_sum_kernel(const float* __restrict__ part, float* __restrict__ dA, float* __restrict__ dD,
                    float* __restrict__ dbias, int b, int H, int nc)
{
    __shared__ float red[3][256];
    const int h = blockIdx.x, tid = threadIdx.x;
    const size_t per_chain = (size_t)nc * kParts;
    const size_t nparts = (size_t)b * H * per_chain;
    float a = 0.0f, d = 0.0f, s = 0.0f;
    for (int bi = 0; bi < b; ++bi) {
        const size_t o = (size_t)(bi * H + h) * per_chain;
        for (size_t k = tid; k < per_chain; k += 256) {
            a += part[o + k];
            d += part[nparts + o + k];
            s += part[2 * nparts + o + k];
        }
    }
    red[0][tid] = a;
    red[1][tid] = d;
    red[2][tid] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (tid < w) {
            red[0][tid] += red[0][tid + w];
            red[1][tid] += red[1][tid + w];
            red[2][tid] += red[2][tid + w];
        }
        __syncthreads();
    }
    if (tid == 0) {
        dA[h] = red[0][0];
        dD[h] = red[1][0];
        dbias[h] = red[2][0];
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qr{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

// 3-D bf16 map: dim0 channels (contiguous), dim1 rows (row_bytes apart),
// dim2 sequences (rows * row_bytes apart); box 64 x 128 x 1, 128-byte
// swizzle; rows past the end read as zero.
cudaError_t map3d(CUtensorMap* m, const void* base, uint64_t channels, uint64_t rows, uint64_t seqs,
                  uint64_t row_bytes)
{
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {channels, rows, seqs};
    const cuuint64_t strides[2] = {row_bytes, row_bytes * rows};
    const cuuint32_t box[3] = {64, (cuuint32_t)kQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t al256(size_t n) { return (n + 255) / 256 * 256; }

struct TcWs {
    size_t ctrl, S, dS, hb, gb, cl, part, total;
};

TcWs tc_ws_layout(int b, int L, int H)
{
    const size_t chains = (size_t)b * H;
    const size_t nc = (size_t)(L + kQ - 1) / kQ;
    TcWs w{};
    size_t o = 0;
    w.ctrl = o;
    o += 256;
    w.S = o;
    o += al256(chains * nc * kStatesDim * 2);
    w.dS = o;
    o += al256(chains * nc * kStatesDim * 2);
    w.hb = o;
    o += al256(chains * nc * kStatesDim * 2);
    w.gb = o;
    o += al256(chains * nc * kStatesDim * 2);
    w.cl = o;
    o += al256(chains * nc * 4);
    w.part = o;
    o += al256(3 * chains * nc * kParts * 4);
    w.total = o;
    return w;
}

bool a16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

}  // namespace

bool scan_bwd_tc_shape(int P, int N, bool bf16) { return bf16 && P == kP && N == kN; }

bool scan_bwd_tc_supported(const ScanBwdArgs& a)
{
    return scan_bwd_tc_shape(a.P, a.N, a.bf16) && a.b > 0 && a.L > 0 && (int64_t)a.b * a.G < 65536 &&
           a.H / a.G <= kMaxHpg &&
           a.row_stride % 8 == 0 && a16(a.x) &&
           a16(a.B) && a16(a.C) && a16(a.dy) && a16(a.dx) && a16(a.dB) && a16(a.dC) && a16(a.workspace) &&
           (size_t)a.b * a.H * ((a.L + kQ - 1) / kQ) * kN < 0x7fffffffULL;
}

size_t scan_bwd_tc_workspace_bytes(int b, int L, int H)
{
    if (b <= 0 || L <= 0) return 0;
    return tc_ws_layout(b, L, H).total;
}

cudaError_t launch_scan_bwd_tc(const ScanBwdArgs& a, cudaStream_t s)
{
    const int nc = (a.L + kQ - 1) / kQ;
    const TcWs w = tc_ws_layout(a.b, a.L, a.H);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    TcParams p{};
    p.dt_raw = static_cast<const __nv_bfloat16*>(a.dt_raw);
    p.dy = static_cast<const __nv_bfloat16*>(a.dy);
    p.x = static_cast<const __nv_bfloat16*>(a.x);
    p.row_stride = a.row_stride;
    p.dt_bias = a.dt_bias;
    p.A = a.A;
    p.D = a.D;
    p.init_state = a.init_state;
    p.dfinal = a.dfinal;
    p.dx = static_cast<__nv_bfloat16*>(a.dx);
    p.dB = static_cast<__nv_bfloat16*>(a.dB);
    p.dC = static_cast<__nv_bfloat16*>(a.dC);
    p.ddt_raw = static_cast<__nv_bfloat16*>(a.ddt_raw);
    p.dA = a.dA;
    p.dD = a.dD;
    p.ddt_bias = a.ddt_bias;
    p.dinit = a.dinit;
    p.status = reinterpret_cast<int32_t*>(ws + w.ctrl);
    p.ws_S = reinterpret_cast<__nv_bfloat16*>(ws + w.S);
    p.ws_dS = reinterpret_cast<__nv_bfloat16*>(ws + w.dS);
    p.ws_hb = reinterpret_cast<__nv_bfloat16*>(ws + w.hb);
    p.ws_gb = reinterpret_cast<__nv_bfloat16*>(ws + w.gb);
    p.ws_cl = reinterpret_cast<float*>(ws + w.cl);
    p.ws_part = reinterpret_cast<float*>(ws + w.part);
    p.b = a.b;
    p.L = a.L;
    p.H = a.H;
    p.G = a.G;
    p.nc = nc;

    const uint64_t rb = (uint64_t)a.row_stride * 2;
    const uint64_t state_rows = (uint64_t)a.b * a.H * nc * kN;
    CUtensorMap tmX, tmB, tmC, tmDY, tmHb, tmGb, tmS, tmdS;
    cudaError_t e;
    if ((e = map3d(&tmX, a.x, (uint64_t)a.H * kP, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = map3d(&tmB, a.B, (uint64_t)a.G * kN, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = map3d(&tmC, a.C, (uint64_t)a.G * kN, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = map3d(&tmDY, a.dy, (uint64_t)a.H * kP, a.L, a.b, (uint64_t)a.H * kP * 2)) != cudaSuccess) return e;
    if ((e = map3d(&tmHb, p.ws_hb, kP, state_rows, 1, kP * 2)) != cudaSuccess) return e;
    if ((e = map3d(&tmGb, p.ws_gb, kP, state_rows, 1, kP * 2)) != cudaSuccess) return e;
    if ((e = map3d(&tmS, p.ws_S, kP, state_rows, 1, kP * 2)) != cudaSuccess) return e;
    if ((e = map3d(&tmdS, p.ws_dS, kP, state_rows, 1, kP * 2)) != cudaSuccess) return e;

    if ((e = cudaMemsetAsync(p.status, 0, 4, s)) != cudaSuccess) return e;
    const dim3 grid((unsigned)nc, (unsigned)(a.b * a.G));
    if ((e = cudaFuncSetAttribute(bwd_states_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, k1::kSmemBytes)) !=
        cudaSuccess)
        return e;
    bwd_states_kernel<<<grid, k1::kThreads, k1::kSmemBytes, s>>>(tmX, tmB, tmC, tmDY, tmS, tmdS, p);
    bwd_pass_kernel<<<dim3((unsigned)(a.b * a.H), kPassSlices, 2), kPassThreads, 0, s>>>(p);
    if ((e = cudaFuncSetAttribute(bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, k3::kSmemBytes)) !=
        cudaSuccess)
        return e;
    bwd_chunk_kernel<<<grid, k3::kThreads, k3::kSmemBytes, s>>>(tmX, tmB, tmC, tmDY, tmHb, tmGb, p);
    bwd_head_sum_kernel<<<a.H, 256, 0, s>>>(p.ws_part, a.dA, a.dD, a.ddt_bias, a.b, a.H, nc);
    return cudaGetLastError();
}

}  // namespace ssd
