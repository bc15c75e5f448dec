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
//   G      = C B^T                         (Q x Q, K = N)    tcgen05 -> TMEM
//   M[i,j] = G[i,j] 2^(cl_i - cl_j) dt_j    (j <= i, else 0)  CUDA cores -> smem
//   Yd     = M X                           (Q x P, K = Q)    tcgen05 -> TMEM
//   Yo     = C h_prev^T                    (Q x P, K = N)    tcgen05 -> TMEM
//   h      = 2^(cl_last) h_prev + B^T (w o X),  w_j = 2^(cl_last - cl_j) dt_j
//            (the decay is applied to h in TMEM, then the product accumulates onto it)
//   y_i    = Yd_i + 2^(cl_i) Yo_i + D x_i                    -> bf16
//
// The decay mask is factored per 32-token block: for a column block J
// strictly below row i's block, 2^(cl_i - cl_j) = 2^(cl_i - cl_e) 2^(cl_e - cl_j)
// with e the last token of J, both factors <= 1 (the decay never grows), so
// only the 32 x 32 diagonal blocks need one exponential per element.
//
// CTA = 8 elementwise warps + 1 control warp; two CTAs per SM.  The control
// warp issues the TMA loads (128-byte swizzle, no multicast) and the
// tcgen05.mma batches, and computes the next chunk's dt / cumulative decay
// while the elementwise warps work; the two sides meet only on mbarriers.
// Elementwise warp w serves TMEM lanes 32*(w%4).. (token rows, or state
// columns n) and column half w/4.  The fp32 state lives in TMEM and never
// leaves the chip inside a sequence.
//
// Scheduling is persistent and balanced: the (sequence x head) chains times
// their chunks form one list of units that is cut into equal contiguous
// ranges, one per CTA, taken in ticket order.  A chain cut by a range
// boundary is finished by the next CTA, which starts from the state the
// previous CTA published in the workspace.  Each CTA first runs the
// segment it must publish, last the segment that depends on its
// predecessor, so the hand-off wait is normally zero.  Every wait (mbarrier
// or hand-off flag) is bounded (1 s); a CTA that gives up records
// SSD_ERR_TIMEOUT in the optional status word and runs to its end without
// waiting again.
//
// Token rows past the end of the sequence are zero-filled by TMA and get
// dt = 0, so a ragged last chunk needs no special case.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kQ = 128;          // chunk length
constexpr int kP = 64;           // head dim
constexpr int kN = 128;          // state size
constexpr int kEwThreads = 256;  // 8 elementwise warps: 4 lane quadrants x 2 column halves
constexpr int kThreads = kEwThreads + 32;
constexpr int kCtlWarp = kEwThreads / 32;
constexpr uint32_t kTmemCols = 256;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kEwBarrier = 1;    // named barrier among the elementwise warps
constexpr int kVecBarrier = 2;   // named barrier among elementwise warps 0-3

// Shared-memory layout, offsets from a 1024-byte aligned base.  Tiles are
// 128-byte swizzled: 128-byte rows, 16-byte chunk c of row r at r*128 +
// ((c ^ (r & 7)) * 16).  Tiles 128 elements wide along their contiguous
// dimension are stored as two 16 KB halves (64 elements each).
constexpr int kOffB = 0;              // B tile  [128 tok][128 n]   (2 halves)
constexpr int kOffC = 32768;          // C tile  [128 tok][128 n]   (2 halves), then M [128 i][128 j]
constexpr int kOffX = 65536;          // X tile  [128 tok][64 p]
constexpr int kOffHX = 81920;         // bf16 state [128 n][64 p], then w o X [128 tok][64 p]
constexpr int kOffVec = 98304;        // per chunk parity: cl, dt, v  (3 x float[128]) x 2
constexpr int kOffBar = kOffVec + 3072 + 32;  // (4 warp totals before it) 6 mbarriers
constexpr int kOffMisc = kOffBar + 64;   // tmem slot, abort flag, ticket
constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + alignment slack

constexpr uint32_t kTileHalf = 16384;
constexpr uint32_t kBytesLoad = 5 * 16384;   // B, C (two halves each) and X

// TMEM columns
constexpr uint32_t kColG = 0;     // G [0,128), then Yd [0,64)
constexpr uint32_t kColYo = 128;  // Yo [128,192)
constexpr uint32_t kColH = 192;   // fp32 state [192,256): lane n, column p

// instruction descriptors
constexpr uint32_t kIdG = umma_idesc_bf16(128, 128, false, false);   // C (K-maj) x B (K-maj)
constexpr uint32_t kIdYo = umma_idesc_bf16(128, 64, false, true);    // C (K-maj) x h (MN-maj)
constexpr uint32_t kIdYd = umma_idesc_bf16(128, 64, false, true);    // M (K-maj) x X (MN-maj)
constexpr uint32_t kIdS = umma_idesc_bf16(128, 64, true, true);      // B^T (MN-maj) x wX (MN-maj)

// Workspace: control block (ticket, hand-off flags), then one published
// fp32 state [P][N] per range boundary.
constexpr size_t kWsCtrlBytes(int slots) { return ((size_t)(64 + 4 * slots) + 255) / 256 * 256; }
constexpr size_t kStateBytes = (size_t)kP * kN * 4;

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

struct ChunkVecs {
    float* cl;   // cumulative log2 decay, inclusive
    float* dt;
    float* v;    // 2^(cl_e - cl_j) dt_j, e = last token of j's 32-block
};

__device__ inline ChunkVecs chunk_vecs(uint8_t* smem, int parity)
{
    float* base = reinterpret_cast<float*>(smem + kOffVec) + parity * 3 * kQ;
    return ChunkVecs{base, base + kQ, base + 2 * kQ};
}

// A CTA's contiguous range of the unit list (chain-major, nc chunks per
// chain), in processing order: A = the head of the last chain (published at
// its end), B = whole chains, C = the tail of the first chain (starts from
// the predecessor's published state).
struct Range {
    int chA, lenA;
    int chB0, chB1;
    int chC, startC;
    int count;
};

__device__ inline Range make_range(int t, int nslots, long long units, int nc)
{
    const long long u0 = units * t / nslots, u1 = units * (t + 1) / nslots;
    Range r;
    const int ch0 = (int)(u0 / nc), c0 = (int)(u0 % nc);
    const int ch1 = (int)(u1 / nc), c1 = (int)(u1 % nc);
    r.chA = ch1;
    r.lenA = c1;
    r.chC = ch0;
    r.startC = c0;
    r.chB0 = c0 > 0 ? ch0 + 1 : ch0;
    r.chB1 = ch1;
    r.count = r.lenA + (r.chB1 - r.chB0) * nc + (c0 > 0 ? nc - c0 : 0);
    return r;
}

struct Item {
    int chain, chunk;
    bool seg_start, seg_end, publish, depend;
};

__device__ inline Item item_at(const Range& r, int idx, int nc)
{
    Item it;
    if (idx < r.lenA) {
        it.chain = r.chA;
        it.chunk = idx;
        it.seg_start = idx == 0;
        it.seg_end = idx == r.lenA - 1;
        it.publish = it.seg_end;
        it.depend = false;
        return it;
    }
    idx -= r.lenA;
    const int nb = (r.chB1 - r.chB0) * nc;
    if (idx < nb) {
        it.chain = r.chB0 + idx / nc;
        it.chunk = idx % nc;
        it.seg_start = it.chunk == 0;
        it.seg_end = it.chunk == nc - 1;
        it.publish = false;
        it.depend = false;
        return it;
    }
    idx -= nb;
    it.chain = r.chC;
    it.chunk = r.startC + idx;
    it.seg_start = idx == 0;
    it.seg_end = it.chunk == nc - 1;
    it.publish = false;
    it.depend = it.seg_start;
    return it;
}

struct Params {
    const __nv_bfloat16* dt_raw;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;
    __nv_bfloat16* y;
    float* final_state;
    int L, H, G, nc, nslots;
    long long units;
    int* ws_ctrl;        // [0] ticket, [16 + t] hand-off flag of boundary t
    float* ws_states;    // [nslots][P][N]
    int32_t* status;
};

__global__ void __launch_bounds__(kThreads, 2)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const Params prm)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + kOffBar);   // TMA B, C, X landed
    uint64_t* bar_m1 = bar_ld + 1;      // G and Yo done
    uint64_t* bar_m2 = bar_ld + 2;      // Yd and the state update done
    uint64_t* bar_mready = bar_ld + 4;  // M, w o X, scaled state ready (elementwise warps)
    uint64_t* bar_hx = bar_ld + 5;      // bf16 state in smem, Yd / Yo consumed (elementwise warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* aborted = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    int* ticket_slot = reinterpret_cast<int*>(smem + kOffMisc + 8);
    uint8_t* sB = smem + kOffB;
    uint8_t* sC = smem + kOffC;   // C, then M
    uint8_t* sX = smem + kOffX;
    uint8_t* sHX = smem + kOffHX; // bf16 state, then w o X
    const uint32_t aB = smem_u32(sB), aC = smem_u32(sC), aX = smem_u32(sX), aHX = smem_u32(sHX);
    const int H = prm.H, nc = prm.nc, L = prm.L;

    if (tid == 0) {
        *aborted = 0;
        mbar_init(bar_ld, 1);
        mbar_init(bar_m1, 1);
        mbar_init(bar_m2, 1);
        mbar_init(bar_mready, kEwThreads);
        mbar_init(bar_hx, kEwThreads);
        fence_mbar_init();
        *ticket_slot = atomicAdd(prm.ws_ctrl, 1);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ticket = *ticket_slot;
    const Range rg = make_range(ticket, prm.nslots, prm.units, nc);

    if (warp == kCtlWarp) {
        // ------------------------------------------------------------------
        // control warp: TMA, MMA issue, chunk vectors
        // ------------------------------------------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmC);
        }
        auto issue_loads = [&](const Item& it) {
            const int bi = it.chain / H, h = it.chain % H, g = h / (H / prm.G);
            const int t0 = it.chunk * kQ;
            mbar_arrive_expect_tx(bar_ld, kBytesLoad);
            tma_load_3d(sB, &tmB, g * kN, t0, bi, bar_ld);
            tma_load_3d(sB + kTileHalf, &tmB, g * kN + 64, t0, bi, bar_ld);
            tma_load_3d(sC, &tmC, g * kN, t0, bi, bar_ld);
            tma_load_3d(sC + kTileHalf, &tmC, g * kN + 64, t0, bi, bar_ld);
            tma_load_3d(sX, &tmX, h * kP, t0, bi, bar_ld);
        };
        if (rg.count > 0 && lane == 0) {
            issue_loads(item_at(rg, 0, nc));
            for (int idx = 0; idx < rg.count; ++idx) {
                const uint32_t ph = (uint32_t)idx & 1u;
                mbar_wait_bounded(bar_ld, ph, kWaitNs, aborted, prm.status);
                mbar_wait_bounded(bar_hx, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)   // G = C B^T
                    umma_bf16(tmem + kColG, desc_kmajor(aC, k), desc_kmajor(aB, k), kIdG, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)   // Yo = C h^T
                    umma_bf16(tmem + kColYo, desc_kmajor(aC, k), desc_mnmajor(aHX, k), kIdYo, k > 0);
                umma_commit(bar_m1);
                mbar_wait_bounded(bar_mready, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)   // Yd = M X
                    umma_bf16(tmem + kColG, desc_kmajor(aC, k), desc_mnmajor(aX, k), kIdYd, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)   // h += B^T (w o X)   (h already decayed)
                    umma_bf16(tmem + kColH, desc_mnmajor(aB, k), desc_mnmajor(aHX, k), kIdS, 1);
                umma_commit(bar_m2);
                mbar_wait_bounded(bar_m2, ph, kWaitNs, aborted, prm.status);
                if (idx + 1 < rg.count) issue_loads(item_at(rg, idx + 1, nc));
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------
        // elementwise warps
        // ------------------------------------------------------------------
        const int quad = warp & 3;          // TMEM lane quadrant
        const int half = warp >> 2;         // column half
        const int row = quad * 32 + lane;   // token row i / state column n
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tG = tmem + kColG, tYd = tmem + kColG, tYo = tmem + kColYo;
        const uint32_t tH = tmem + kColH + (uint32_t)half * 32 + lane_off;

        // start of a segment: fp32 state into TMEM, bf16 copy into smem
        float* sWs = reinterpret_cast<float*>(smem + kOffBar) - 8;   // 4 warp totals
        // dt_raw of token `row` of an item's chunk (warps 0-3)
        auto load_dt = [&](const Item& it) -> float {
            const int t = it.chunk * kQ + row;
            if (half != 0 || t >= L) return 0.0f;
            const int bi = it.chain / H, h = it.chain % H;
            return __bfloat162float(prm.dt_raw[((size_t)bi * L + t) * H + h]);
        };
        // Chunk vectors of an item (warps 0-3, one token each): dt, the
        // inclusive cumulative log2 decay and the off-diagonal column factor.
        // Stage 1 scans within each warp; stage 2, after a barrier among the
        // four warps, adds the preceding warps' totals and writes the vectors.
        float vec_a = 0.0f, vec_dt = 0.0f;
        auto vecs_stage1 = [&](const Item& it, float dtr) {
            const int h = it.chain % H;
            const int t = it.chunk * kQ + row;
            const float bias = prm.dt_bias ? prm.dt_bias[h] : 0.0f;
            vec_dt = t < L ? softplus_f(dtr + bias) : 0.0f;
            vec_a = vec_dt * (prm.A[h] * 1.4426950408889634f);   // dt * A * log2(e)
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, vec_a, o);
                if (lane >= o) vec_a += v;
            }
            if (lane == 31) sWs[quad] = vec_a;
        };
        auto vecs_stage2 = [&](int parity) {
            float pre = 0.0f;
            for (int w = 0; w < quad; ++w) pre += sWs[w];
            const float cl = vec_a + pre;
            const float cl_e = __shfl_sync(0xffffffffu, cl, 31);
            const ChunkVecs cv = chunk_vecs(smem, parity);
            cv.cl[row] = cl;
            cv.dt[row] = vec_dt;
            cv.v[row] = ex2_approx(cl_e - cl) * vec_dt;
        };
        auto make_vecs = [&](const Item& it, float dtr, int parity) {   // warps 0-3 only
            vecs_stage1(it, dtr);
            named_bar_sync(kVecBarrier, 128);
            vecs_stage2(parity);
        };

        // Hand chunk `idx` over to the MMA side (bf16 state in smem, Yd / Yo of
        // the previous chunk consumed); the barrier also publishes the chunk's
        // vectors, written by warps 0-3, to all elementwise warps.
        auto hand_over = [&](int idx) {
            (void)idx;
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar_sync(kEwBarrier, kEwThreads);
            mbar_arrive(bar_hx);
        };
        auto begin_segment = [&](const Item& it, int idx) {
            const int bi = it.chain / H, h = it.chain % H;
            const float* src = nullptr;
            bool cg = false;
            if (it.depend) {
                const int* flag = prm.ws_ctrl + 16 + (ticket - 1);
                if (tid == 0 && !*aborted) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_gpu(flag) == 0) {
                        if (globaltimer_ns() - t0 > kWaitNs) {
                            *aborted = 1;
                            if (prm.status) atomicExch(reinterpret_cast<int*>(prm.status), 4);
                            break;
                        }
                    }
                }
                named_bar_sync(kEwBarrier, kEwThreads);
                src = prm.ws_states + (size_t)(ticket - 1) * (kP * kN);
                cg = true;
            } else if (prm.init_state) {
                src = prm.init_state + ((size_t)bi * H + h) * (size_t)(kP * kN);
            }
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                const int p0 = half * 32 + pc * 16;
                float hv[16];
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    const float* q = src + (size_t)(p0 + p) * kN + row;
                    hv[p] = src ? (cg ? __ldcg(q) : *q) : 0.0f;
                }
                tmem_st16(tH + pc * 16, hv);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    *reinterpret_cast<uint4*>(sHX + sw128(row, (p0 >> 3) + q)) = pack_bf16x8(&hv[q * 8]);
            }
            tmem_wait_st();
            hand_over(idx);
        };

        float dtr_next = 0.0f;
        if (rg.count > 0 && half == 0) {
            make_vecs(item_at(rg, 0, nc), load_dt(item_at(rg, 0, nc)), 0);
            if (rg.count > 1) dtr_next = load_dt(item_at(rg, 1, nc));
        }
        for (int idx = 0; idx < rg.count; ++idx) {
            const uint32_t ph = (uint32_t)idx & 1u;
            const Item it = item_at(rg, idx, nc);
            const int bi = it.chain / H, h = it.chain % H;
            const float Dh = prm.D ? prm.D[h] : 0.0f;
            if (it.seg_start) begin_segment(it, idx);

            mbar_wait_bounded(bar_m1, ph, kWaitNs, aborted, prm.status);
            mbar_wait_bounded(bar_ld, ph, kWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            const ChunkVecs cv = chunk_vecs(smem, (int)ph);
            const float cl_i = cv.cl[row];
            const float cl_last = cv.cl[kQ - 1];

            // x of this thread's row and column half (kept for D x)
            uint4 xraw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) xraw[q] = *reinterpret_cast<const uint4*>(sX + sw128(row, half * 4 + q));

            // M = G o L: row `row`, column blocks {0,3} (half 0) or {1,2} (half 1),
            // written over C (both MMAs reading C are done); 16 columns at a time
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int jb = half == 0 ? (s2 == 0 ? 0 : 3) : (s2 == 0 ? 1 : 2);
                const float u = ex2_approx(cl_i - cv.cl[jb * 32 + 31]);
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const int j0 = jb * 32 + pc * 16;
                    uint4 packed[2];
                    if (jb <= quad) {
                        float gv[16];
                        tmem_ld16(tG + lane_off + j0, gv);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            float m[8];
                            if (jb < quad) {
                                const float4 va = reinterpret_cast<const float4*>(cv.v + j0 + q * 8)[0];
                                const float4 vb = reinterpret_cast<const float4*>(cv.v + j0 + q * 8)[1];
                                const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                                for (int e = 0; e < 8; ++e) m[e] = gv[q * 8 + e] * u * vv[e];
                            } else {
                                const float4 ca = reinterpret_cast<const float4*>(cv.cl + j0 + q * 8)[0];
                                const float4 cb = reinterpret_cast<const float4*>(cv.cl + j0 + q * 8)[1];
                                const float4 da = reinterpret_cast<const float4*>(cv.dt + j0 + q * 8)[0];
                                const float4 db = reinterpret_cast<const float4*>(cv.dt + j0 + q * 8)[1];
                                const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                                const float dd[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
                                for (int e = 0; e < 8; ++e) {
                                    const int j = j0 + q * 8 + e;
                                    const float v = gv[q * 8 + e] * ex2_approx(cl_i - cc[e]) * dd[e];
                                    m[e] = (j <= row) ? v : 0.0f;
                                }
                            }
                            packed[q] = pack_bf16x8(m);
                        }
                    } else {
                        packed[0] = packed[1] = make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int jq = j0 + q * 8;
                        *reinterpret_cast<uint4*>(sC + (jq >> 6) * kTileHalf + sw128(row, (jq & 63) >> 3)) = packed[q];
                    }
                }
            }
            // w o X over the bf16 state copy (C h^T, its reader, is done)
            {
                const float wj = ex2_approx(cl_last - cl_i) * cv.dt[row];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float v[8];
                    unpack_bf16x8(xraw[q], v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] *= wj;
                    *reinterpret_cast<uint4*>(sHX + sw128(row, half * 4 + q)) = pack_bf16x8(v);
                }
            }
            // decay the fp32 state in place; the chunk-state product accumulates onto it
            {
                const float decay = ex2_approx(cl_last);
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    float hv[16];
                    tmem_ld16(tH + pc * 16, hv);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 16; ++p) hv[p] *= decay;
                    tmem_st16(tH + pc * 16, hv);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_mready);
            // the next chunk's vectors while the tensor cores run (its parity
            // buffer was last read in chunk idx-1, which every warp has left)
            if (half == 0 && idx + 1 < rg.count) {
                make_vecs(item_at(rg, idx + 1, nc), dtr_next, (idx + 1) & 1);
                if (idx + 2 < rg.count) dtr_next = load_dt(item_at(rg, idx + 2, nc));
            }

            mbar_wait_bounded(bar_m2, ph, kWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            // new state: bf16 copy for the next chunk, or out at the end of a segment
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                float hv[16];
                tmem_ld16(tH + pc * 16, hv);
                tmem_wait_ld();
                const int p0 = half * 32 + pc * 16;
                if (!it.seg_end) {
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        *reinterpret_cast<uint4*>(sHX + sw128(row, (p0 >> 3) + q)) = pack_bf16x8(&hv[q * 8]);
                } else if (it.publish) {
                    float* dst = prm.ws_states + (size_t)ticket * (kP * kN);
#pragma unroll
                    for (int p = 0; p < 16; ++p) __stcg(dst + (size_t)(p0 + p) * kN + row, hv[p]);
                } else if (prm.final_state) {
                    float* dst = prm.final_state + ((size_t)bi * H + h) * (size_t)(kP * kN);
#pragma unroll
                    for (int p = 0; p < 16; ++p) dst[(size_t)(p0 + p) * kN + row] = hv[p];
                }
            }
            if (it.seg_end && it.publish) {
                __threadfence();
                named_bar_sync(kEwBarrier, kEwThreads);
                if (tid == 0) st_release_gpu(prm.ws_ctrl + 16 + ticket, 1);
            }
            // output: y = Yd + 2^cl Yo + D x, token row `row`, p of this half
            {
                const int t = it.chunk * kQ + row;
                const float sc = ex2_approx(cl_i);
                __nv_bfloat16* yrow = prm.y + (((size_t)bi * L + t) * H + h) * kP + half * 32;
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    float yd[16], yo[16];
                    tmem_ld16(tYd + lane_off + half * 32 + pc * 16, yd);
                    tmem_ld16(tYo + lane_off + half * 32 + pc * 16, yo);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        float xv[8], o[8];
                        unpack_bf16x8(xraw[pc * 2 + q], xv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = yd[q * 8 + e] + sc * yo[q * 8 + e] + Dh * xv[e];
                        if (t < L) *reinterpret_cast<uint4*>(yrow + pc * 16 + q * 8) = pack_bf16x8(o);
                    }
                }
            }
            // hand Yd / Yo and the bf16 state over to the next chunk's MMAs;
            // a new segment hands over after loading its initial state
            if (idx + 1 < rg.count && !it.seg_end) hand_over(idx + 1);
        }
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


int tc_slots(const ScanArgs& a)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    const long long chains = (long long)a.b * a.H;
    const long long slots = 2LL * sms;   // two CTAs per SM
    return (int)(chains < slots ? chains : slots);
}

}  // namespace

bool chunk_scan_tc_supported(const ScanArgs& a)
{
    return a.bf16 && a.P == kP && a.N == kN && a.Q == kQ;
}

size_t chunk_scan_tc_workspace_bytes(const ScanArgs& a)
{
    if (a.b <= 0 || a.L <= 0) return 0;
    const int slots = tc_slots(a);
    return kWsCtrlBytes(slots) + (size_t)slots * kStateBytes;
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
    const int slots = tc_slots(a);
    const size_t ctrl = kWsCtrlBytes(slots);
    if (!a.workspace || a.workspace_bytes < ctrl + (size_t)slots * kStateBytes) return cudaErrorInvalidValue;
    // ticket counter and hand-off flags start at zero on every call
    if ((e = cudaMemsetAsync(a.workspace, 0, ctrl, s)) != cudaSuccess) return e;
    Params prm;
    prm.dt_raw = static_cast<const __nv_bfloat16*>(a.dt_raw);
    prm.dt_bias = a.dt_bias;
    prm.A = a.A;
    prm.D = a.D;
    prm.init_state = a.init_state;
    prm.y = static_cast<__nv_bfloat16*>(a.y);
    prm.final_state = a.final_state;
    prm.L = a.L;
    prm.H = a.H;
    prm.G = a.G;
    prm.nc = (a.L + kQ - 1) / kQ;
    prm.nslots = slots;
    prm.units = (long long)a.b * a.H * prm.nc;
    prm.ws_ctrl = static_cast<int*>(a.workspace);
    prm.ws_states = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + ctrl);
    prm.status = a.status;
    chunk_scan_tc_kernel<<<slots, kThreads, kSmemBytes, s>>>(tmX, tmB, tmC, prm);
    return cudaGetLastError();
}

}  // namespace ssd
