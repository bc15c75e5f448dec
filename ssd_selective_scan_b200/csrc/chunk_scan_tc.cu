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
//   M[i,j] = G[i,j] 2^(cl_i - cl_j) dt_j    (j < i)
//          = G[i,i] dt_i + D                (j = i), 0 (j > i)  CUDA cores -> TMEM
//   Yd     = M X                           (Q x P, K = Q)    tcgen05 (A from TMEM)
//   Yo     = C h_prev^T                    (Q x P, K = N)    tcgen05 -> TMEM
//   h      = 2^(cl_last) h_prev + B^T (w o X),  w_j = 2^(cl_last - cl_j) dt_j
//            (the decay is applied to h in TMEM, then the product accumulates onto it)
//   y_i    = Yd_i + 2^(cl_i) Yo_i                            -> bf16
// (D on M's diagonal makes M X include the skip term D x.)
//
// The decay mask is factored per 32-token block: for a column block J
// strictly below row i's block, 2^(cl_i - cl_j) = 2^(cl_i - cl_e) 2^(cl_e - cl_j)
// with e the last token of J, both factors <= 1 (the decay never grows), so
// only the 32 x 32 diagonal blocks need one exponential per element.
//
// CTA = 16 elementwise warps + an MMA warp + a producer warp + a vector
// warp, one CTA per SM, software-pipelined across chunks.  The producer warp
// issues the TMA loads (128-byte swizzle, no multicast) into two stages one
// chunk ahead and stores each chunk's y tile by TMA; the vector warp computes
// the next chunk's dt / cumulative decay vectors, its dt loads issued a chunk
// earlier still.  The MMA warp only waits and issues tcgen05.mma (issue
// blocks until the tensor core accepts the instruction, so nothing else may
// sit on that thread).  Per chunk the elementwise warps first release the
// state products (bf16 state copy, decayed state, w o X), then finish the
// previous chunk's y while those run, then build the masked tile, after
// which M X and the next chunk's C B^T run.  The warps meet only on
// mbarriers, each waiter gated by what it waits for, so no barrier runs two
// phases ahead of a waiter.
// Elementwise warp w serves TMEM lanes 32*(w%4).. (token rows, or state
// columns n) and column quarter w/4.  The fp32 state lives in TMEM and never
// leaves the chip inside a sequence.
//
// Scheduling is persistent and balanced: the (sequence x head) chains times
// their chunks form one list of units that is cut into equal contiguous
// ranges, one per CTA, taken in ticket order.  A chain cut by a range
// boundary is finished by the next CTA, which starts from the state the
// previous CTA published in the workspace.  Each CTA first runs the
// segment it must publish, last the segment that depends on its
// predecessor, so the hand-off wait is normally zero.  Every wait is
// bounded: an mbarrier wait by 1 s, a hand-off wait by 1 s plus 16 us per
// chunk of the chain before the range; a CTA that gives up records
// SSD_ERR_TIMEOUT in the optional status word and runs to its end without
// waiting again.
//
// Long chains (fewer chains than SMs, e.g. one 262144-token sequence of 64
// heads): every chain is cut into equal ranges, s per chain for s * chains
// <= SMs, and a CTA whose range starts inside a chain rebuilds its starting
// state itself instead of waiting for the CTA before it.  The state entering
// chunk c0 is sum over earlier chunks c of 2^(decay from c's end to c0) S_c,
// plus the initial state decayed from the chain's start.  Walking back over
// at most kPreMax chunks, the decay 2^(sum of cl_last) from the end of each
// one to c0 is folded into its weights, w'_j = 2^(Lrun + cl_last - cl_j) dt_j,
// so all of them accumulate into one TMEM accumulator, S += B^T (w' o X),
// with no per-chunk decay step (the "state-only" items: B and X loaded, no
// C, no y).  If the walk reaches the chain's start, the decayed initial
// state is added; if instead the accumulated decay has fallen below 2^-64,
// older tokens weigh less than 2^-64 of their own size, far under float32
// rounding, and are dropped.  Otherwise (a long-memory head) the CTA falls
// back to the published state of its predecessor.
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
constexpr int kEwWarps = 16;     // elementwise warps: 4 lane quadrants x 4 column quarters
constexpr int kEwThreads = kEwWarps * 32;
constexpr int kMmaWarp = kEwWarps;       // issues tcgen05.mma
constexpr int kProdWarp = kEwWarps + 1;  // TMA loads / stores
constexpr int kVecWarp = kEwWarps + 2;   // chunk vectors (dt, cumulative decay)
constexpr int kThreads = kEwThreads + 96;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint64_t kWaitPerChunkNs = 16000;   // hand-off waits: + 16 us per chunk before the range
constexpr int kPreMax = 32;            // chunks a range's starting state is rebuilt from, at most
constexpr int kMinRangeLong = 32;      // units per CTA at least, when chains are split across CTAs
constexpr float kPreCutLog2 = -64.0f;  // accumulated log2 decay below which older tokens are dropped
constexpr int kEwBarrier = 1;    // named barrier among the elementwise warps

// Shared-memory layout, offsets from a 1024-byte aligned base.  Tiles are
// 128-byte swizzled: 128-byte rows, 16-byte chunk c of row r at r*128 +
// ((c ^ (r & 7)) * 16).  Tiles 128 elements wide along their contiguous
// dimension are stored as two 16 KB halves (64 elements each).
constexpr int kStageBytes = 81920;    // B [128 tok][128 n], C [128 tok][128 n], X [128 tok][64 p]
constexpr int kOffStage = 0;          // 2 stages
constexpr int kStB = 0, kStC = 32768, kStX = 65536;
constexpr int kOffHB = 2 * kStageBytes;         // bf16 state entering the item [128 n][64 p]
constexpr int kOffWX = kOffHB + 16384;          // w o X [128 tok][64 p]
constexpr int kOffVec = kOffWX + 16384;         // per chunk parity: cl, dt, v  (3 x float[128]) x 2
constexpr int kMaxSeqSmem = 1024;               // ragged batches: tables in shared memory up to this
constexpr int kOffSeq = kOffVec + 3072;         // cu_seqlens, then seq_units (int[kMaxSeqSmem + 1] each)
constexpr int kOffBar = kOffSeq + 8 * (kMaxSeqSmem + 1) + 8;   // mbarriers (8-byte aligned)
constexpr int kNumBars = 13;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;   // tmem slot, abort flag, ticket
constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + alignment slack

constexpr uint32_t kTileHalf = 16384;
constexpr uint32_t kBytesBC = 4 * 16384;   // B and C, two halves each
constexpr uint32_t kBytesX = 16384;

// TMEM columns
constexpr uint32_t kColG = 0;     // G [0,128)
constexpr uint32_t kColM = 128;   // masked tile M, bf16 pairs along j [128,192)
constexpr uint32_t kColYd = 192;  // Yd [192,256)
constexpr uint32_t kColYo = 256;  // Yo, two buffers [256,320) and [320,384)
constexpr uint32_t kColH = 384;   // fp32 state [384,448): lane n, column p

// instruction descriptors
constexpr uint32_t kIdG = umma_idesc_bf16(128, 128, false, false);   // C (K-maj) x B (K-maj)
constexpr uint32_t kIdYo = umma_idesc_bf16(128, 64, false, true);    // C (K-maj) x h (MN-maj)
constexpr uint32_t kIdYd = umma_idesc_bf16(128, 64, false, true);    // M (TMEM, K-maj) x X (MN-maj)
constexpr uint32_t kIdS = umma_idesc_bf16(128, 64, true, true);      // B^T (MN-maj) x wX (MN-maj)

// Workspace: control block (ticket, hand-off flags), then one published
// fp32 state [P][N] per range boundary.
constexpr size_t kWsCtrlBytes(int slots) { return ((size_t)(64 + 4 * slots) + 255) / 256 * 256; }
constexpr size_t kStateBytes = (size_t)kP * kN * 4;

// softplus(v) = max(v, 0) + log(1 + e^-|v|) with the hardware exp and log
// (bf16 outputs: well inside their rounding; for v < -17 the log term
// rounds to 0, i.e. dt below 4e-8 becomes 0).
__device__ inline float softplus_fast(float v)
{
    return fmaxf(v, 0.0f) + __logf(1.0f + __expf(-fabsf(v)));
}

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

// Eight bf16 values times w, in bf16 pairs: w is rounded to bf16 once
// (relative error 2^-9, like the product's own rounding), then each product
// is rounded to bf16 as the packed fp32 form did.  Half the instructions of
// unpack, fp32 multiply and pack.
__device__ inline uint4 scale_bf16x8(uint4 q, __nv_bfloat162 w)
{
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __hmul2(h[i], w);
    return q;
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

// Division by a runtime constant d (1 <= d < 2^31) as a multiply-high and
// a shift (round-up reciprocal method for 32-bit unsigned division).
struct FastDiv {
    uint32_t d, m, s;
    __host__ static FastDiv make(uint32_t d)
    {
        FastDiv f;
        f.d = d;
        f.s = 0;
        while ((1ull << f.s) < d) ++f.s;
        f.m = (uint32_t)((((1ull << 32) * ((1ull << f.s) - d)) / d) + 1);
        return f;
    }
    __device__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

struct Params {
    const __nv_bfloat16* dt_raw;
    const float* dt_bias;
    const float* A;
    const float* D;
    const float* init_state;
    __nv_bfloat16* y;
    float* final_state;
    int L, H, G, nc, nslots;   // L: tokens per sequence (dense) or in the packed dimension (ragged)
    int Hf;                    // heads per sequence (H counts head pairs in the pair kernel)
    int units;                 // dense batches: units in the list
    FastDiv fnc, fH, fHG;      // division by nc, H, H / G
    int* ws_ctrl;        // [0] ticket, [16 + t] hand-off flag of boundary t
    float* ws_states;    // [nslots][P][N]
    int32_t* status;
    // Ragged batches (cu_seqlens != nullptr): sequence s is the packed tokens
    // cu_seqlens[s] .. cu_seqlens[s+1] - 1; seq_units[s] = H times the chunk
    // count of the sequences before s; ws_hdr[0] != 0 marks an invalid
    // cu_seqlens (nothing is done), ws_hdr[1] = the number of units.
    const int* cu_seqlens;
    const int* seq_units;
    const int* ws_hdr;
    int4* unit_desc;         // per unit: {chain, chunk, first token, end of its sequence}
    int nseq;
};

// The unit list: chains c = s * H + h (sequence-major), each the chunks of
// its sequence in order.  Unit u -> (chain, chunk, chunks in that chain).
struct Loc {
    int chain, chunk, ncc;
};

// Ragged batches' tables, in shared memory when they fit (else global):
// cu = cu_seqlens, su = seq_units.
struct Tabs {
    const int* cu;
    const int* su;
    const int4* desc;   // per-unit descriptors (global memory)
};

// A unit descriptor written earlier in this kernel by this CTA (a plain
// coherent load, never the read-only path).
__device__ inline int4 ld_desc(const int4* p)
{
    int4 v;
    asm volatile("ld.global.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// `hint` is a sequence at or before u's; callers that visit units in
// increasing order keep it and the search costs O(1) per call.
template <bool kRagged>
__device__ inline Loc locate(const Params& p, const Tabs& tb, int u, int& hint)
{
    Loc l;
    if constexpr (!kRagged) {
        const int ch = (int)p.fnc.div((uint32_t)u);
        l.chain = ch;
        l.chunk = u - ch * p.nc;
        l.ncc = p.nc;
        return l;
    }
    int s = hint;
    while (s + 1 < p.nseq && tb.su[s + 1] <= u) ++s;
    hint = s;
    const int base = tb.su[s];
    const int ncs = max(1, (tb.su[s + 1] - base) / p.H);   // (never an empty sequence)
    const int local = u - base;
    const int h = local / ncs;
    l.chain = s * p.H + h;
    l.chunk = local - h * ncs;
    l.ncc = ncs;
    return l;
}

// The (non-empty) sequence holding unit u of a ragged batch: the last s
// with seq_units[s] <= u (binary search).
__device__ inline int seq_of_unit(const Params& p, const Tabs& tb, int u)
{
    int lo = 0, hi = p.nseq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.su[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// A CTA's contiguous range of the unit list, in processing order:
//   A = the head of the chain the range ends in (published at its end);
//   B = whole chains;
//   C = the tail of the chain the range starts in, from the predecessor's
//       published state.
// A range that starts and ends inside one chain is a single C segment that
// is published at its end too.
//   P = (long chains only) npre state-only items, chunks startC - 1 down to
//       startC - npre of chain chC, run just before C to rebuild its
//       starting state.
struct Range {
    int chA, lenA;
    int uB0, nB, sB0;   // B: units [uB0, uB0 + nB); sB0 = sequence of uB0
    int uA0, uC0;       // first units of A and of C (C's state-only items precede uC0)
    int uEnd;           // one past the range's last unit
    int chC, startC, lenC;
    bool pubC;
    int npre;           // state-only items before C
    int count;
    __device__ int pre_begin() const { return lenA + nB; }
    __device__ bool is_pre(int idx) const { return idx >= lenA + nB && idx < lenA + nB + npre; }
};

template <bool kRagged, bool kLong>
__device__ inline Range make_range(const Params& p, const Tabs& tb, int t, int units)
{
    Range r{};
    const int u0 = (int)((long long)units * t / p.nslots);
    const int u1 = (int)((long long)units * (t + 1) / p.nslots);
    if (u1 <= u0) return r;
    int hint0 = kRagged ? seq_of_unit(p, tb, u0) : 0;
    const Loc a = locate<kRagged>(p, tb, u0, hint0);
    Loc b{-1, 0, 0};   // u1 == units: the end of the list
    if (u1 < units) {
        int hint1 = kRagged ? seq_of_unit(p, tb, u1) : 0;
        b = locate<kRagged>(p, tb, u1, hint1);
    }
    r.uC0 = u0;
    r.uEnd = u1;
    if (a.chunk > 0 && b.chain == a.chain) {   // inside one chain
        r.chC = a.chain;
        r.startC = a.chunk;
        r.lenC = b.chunk - a.chunk;
        r.pubC = true;
        r.npre = kLong ? min(r.startC, kPreMax) : 0;
        r.count = r.npre + r.lenC;
        return r;
    }
    r.chA = b.chain;
    r.lenA = b.chunk;
    r.uA0 = u1 - b.chunk;
    if (a.chunk > 0) {
        r.chC = a.chain;
        r.startC = a.chunk;
        r.lenC = a.ncc - a.chunk;
    }
    r.uB0 = a.chunk > 0 ? u0 + (a.ncc - a.chunk) : u0;
    r.nB = (u1 - b.chunk) - r.uB0;
    r.sB0 = kRagged && r.nB > 0 ? seq_of_unit(p, tb, r.uB0) : 0;
    r.npre = kLong && r.lenC > 0 ? min(r.startC, kPreMax) : 0;
    r.count = r.lenA + r.nB + r.npre + r.lenC;
    return r;
}

struct Item {
    int chain, chunk;
    int seq, h;        // chain = seq * H + h
    int tok0;          // first token of the chunk along the token dimension
    int nvalid;        // tokens of the sequence in the chunk (<= kQ)
    int bi;            // coordinate along the batch dimension (0 for a ragged batch)
    bool seg_start, seg_end, publish, depend;
    bool direct_y;     // y written row by row (a ragged batch's last, partial chunk)
    bool pre;          // state-only item (long chains): rebuilds C's starting state
    bool pre_first, pre_last;
};

template <bool kRagged, bool kLong>
__device__ inline Item item_at(const Params& p, const Tabs& tb, const Range& r, int idx, int& hint)
{
    Item it;
    it.pre = it.pre_first = it.pre_last = false;
    if constexpr (kRagged) {
        // the item's unit, then its descriptor
        int u;
        it.publish = it.depend = false;
        if (idx < r.lenA) {
            u = r.uA0 + idx;
            it.seg_start = idx == 0;
            it.seg_end = it.publish = idx == r.lenA - 1;
        } else if (idx - r.lenA < r.nB) {
            u = r.uB0 + (idx - r.lenA);
        } else if (kLong && idx - r.lenA - r.nB < r.npre) {
            const int k = idx - r.lenA - r.nB;   // walking back from chunk startC - 1
            u = r.uC0 - 1 - k;
            it.seg_start = it.seg_end = false;
            it.pre = true;
            it.pre_first = k == 0;
            it.pre_last = k == r.npre - 1;
        } else {
            const int k = idx - r.lenA - r.nB - r.npre;
            u = r.uC0 + k;
            it.seg_start = it.depend = k == 0;
            it.seg_end = k == r.lenC - 1;
            it.publish = it.seg_end && r.pubC;
        }
        const int4 d = ld_desc(tb.desc + u);   // (written by this CTA in its prologue)
        it.chain = d.x;
        it.chunk = d.y;
        it.tok0 = d.z;
        it.nvalid = min(kQ, d.w - d.z);
        if (idx >= r.lenA && idx - r.lenA < r.nB) {   // B: whole chains
            it.seg_start = d.y == 0;
            it.seg_end = d.w - d.z <= kQ;
        }
        it.seq = (int)p.fH.div((uint32_t)it.chain);
        it.h = it.chain - it.seq * p.H;
        it.bi = 0;
        it.direct_y = it.nvalid < kQ;
        (void)hint;
        return it;
    }
    if (idx < r.lenA) {
        it.chain = r.chA;
        it.chunk = idx;
        it.seg_start = idx == 0;
        it.seg_end = idx == r.lenA - 1;
        it.publish = it.seg_end;
        it.depend = false;
    } else if (idx - r.lenA < r.nB) {
        const Loc l = locate<kRagged>(p, tb, r.uB0 + (idx - r.lenA), hint);
        it.chain = l.chain;
        it.chunk = l.chunk;
        it.seg_start = l.chunk == 0;
        it.seg_end = l.chunk == l.ncc - 1;
        it.publish = false;
        it.depend = false;
    } else if (kLong && idx - r.lenA - r.nB < r.npre) {
        const int k = idx - r.lenA - r.nB;   // walking back from chunk startC - 1
        it.chain = r.chC;
        it.chunk = r.startC - 1 - k;
        it.seg_start = it.seg_end = it.publish = it.depend = false;
        it.pre = true;
        it.pre_first = k == 0;
        it.pre_last = k == r.npre - 1;
    } else {
        const int k = idx - r.lenA - r.nB - r.npre;
        it.chain = r.chC;
        it.chunk = r.startC + k;
        it.seg_start = k == 0;
        it.depend = it.seg_start;
        it.seg_end = k == r.lenC - 1;
        it.publish = it.seg_end && r.pubC;
    }
    it.seq = (int)p.fH.div((uint32_t)it.chain);
    it.h = it.chain - it.seq * p.H;
    if constexpr (kRagged) {
        const int s0 = tb.cu[it.seq];
        const int len = tb.cu[it.seq + 1] - s0;
        it.tok0 = s0 + it.chunk * kQ;
        it.nvalid = min(kQ, len - it.chunk * kQ);
        it.bi = 0;
        it.direct_y = it.nvalid < kQ;
    } else {
        it.tok0 = it.chunk * kQ;
        it.nvalid = min(kQ, p.L - it.tok0);
        it.bi = it.seq;
        it.direct_y = false;
    }
    return it;
}

__device__ inline void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// y tensor maps with boxes of 64, 32, 16 and 8 rows: a ragged batch's
// partial last chunk stores its first rows (a multiple of 8) with at most
// four of them, never reaching the next sequence's rows.
struct YBoxes {
    CUtensorMap m[4];
};

// kLong: ranges inside chains rebuild their starting state (state-only
// items); without it that code is compiled out.
template <bool kRagged, bool kLong>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
                     const __grid_constant__ YBoxes ypart, const Params prm)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* bar_ld = bars + 0;        // [2]: stage's B and C landed (TMA)
    uint64_t* bar_m1 = bars + 2;        // G ready
    uint64_t* bar_m2 = bars + 3;        // Yd ready (all MMAs of the item done)
    uint64_t* bar_sready = bars + 4;    // bf16 state, w o X and decayed state ready (elementwise warps)
    uint64_t* bar_mready = bars + 5;    // masked tile M in TMEM; G, Yd, Yo of earlier items read (elementwise warps)
    uint64_t* bar_vec = bars + 6;       // chunk vectors published (vector warp)
    uint64_t* bar_ldx = bars + 7;       // [2]: stage's X landed (TMA)
    // Per stage, so that the producer warp, which nothing else waits for,
    // can never fall two phases behind them:
    uint64_t* bar_ystaged = bars + 9;   // [2]: y tile staged in the stage's X buffer (elementwise warps)
    uint64_t* bar_m4 = bars + 11;       // [2]: C h^T and the state update done; stage's B and C free
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* aborted = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    int* ticket_slot = reinterpret_cast<int*>(smem + kOffMisc + 8);
    uint8_t* sHB = smem + kOffHB;
    uint8_t* sWX = smem + kOffWX;
    const int H = prm.H, L = prm.L;

    if (tid == 0) {
        *aborted = 0;
        mbar_init(bar_ld, 1);
        mbar_init(bar_ld + 1, 1);
        mbar_init(bar_m1, 1);
        mbar_init(bar_m2, 1);
        mbar_init(bar_sready, kEwThreads);
        mbar_init(bar_mready, kEwThreads);
        mbar_init(bar_vec, 1);
        mbar_init(bar_ldx, 1);
        mbar_init(bar_ldx + 1, 1);
        mbar_init(bar_ystaged, kEwThreads);
        mbar_init(bar_ystaged + 1, kEwThreads);
        mbar_init(bar_m4, 1);
        mbar_init(bar_m4 + 1, 1);
        fence_mbar_init();
        *ticket_slot = atomicAdd(prm.ws_ctrl, 1);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ticket = *ticket_slot;
    // a ragged batch reads its unit count (0 if cu_seqlens was invalid)
    const int units = kRagged ? (prm.ws_hdr[0] ? 0 : prm.ws_hdr[1]) : prm.units;
    Tabs tabs{prm.cu_seqlens, prm.seq_units, prm.unit_desc};
    if constexpr (kRagged) {
        // the ragged tables into shared memory when they fit
        if (prm.nseq <= kMaxSeqSmem && units > 0) {
            int* scu = reinterpret_cast<int*>(smem + kOffSeq);
            int* ssu = scu + (kMaxSeqSmem + 1);
            for (int i = tid; i <= prm.nseq; i += kThreads) {
                scu[i] = prm.cu_seqlens[i];
                ssu[i] = prm.seq_units[i];
            }
            __syncthreads();
            tabs = Tabs{scu, ssu, prm.unit_desc};
        }
    }
    const Range rg = make_range<kRagged, kLong>(prm, tabs, ticket, units);
    if constexpr (kRagged) {
        // the descriptors of this range's units (its state-only items'
        // included), so that every role finds an item with one load; a
        // unit shared with the range before is written by both CTAs with
        // the same value
        if (rg.count > 0) {
            for (int u = rg.uC0 - rg.npre + tid; u < rg.uEnd; u += kThreads) {
                const int sq = seq_of_unit(prm, tabs, u);
                const int base = tabs.su[sq];
                const int ncs = (tabs.su[sq + 1] - base) / prm.H;
                const int h = (u - base) / ncs;
                const int c = u - base - h * ncs;
                prm.unit_desc[u] = make_int4(sq * prm.H + h, c, tabs.cu[sq] + c * kQ, tabs.cu[sq + 1]);
            }
        }
        __syncthreads();
    }
    auto group_of = [&](const Item& it) { return (int)prm.fHG.div((uint32_t)it.h); };
    auto stage = [&](int idx) { return smem + kOffStage + (idx & 1) * kStageBytes; };

    if (warp == kMmaWarp) {
        // ------------------------------------------------------------------
        // MMA warp (one thread): waits and tcgen05.mma issue only
        // ------------------------------------------------------------------
        if (lane == 0 && rg.count > 0) {
            // Stage 1 is kStageBytes after stage 0, so its descriptors are
            // stage 0's plus a constant; selected without indexing.
            const uint32_t st0 = smem_u32(smem + kOffStage);
            const uint64_t dCk0 = desc_kmajor(st0 + kStC, 0), dBk0 = desc_kmajor(st0 + kStB, 0);
            const uint64_t dBmn0 = desc_mnmajor(st0 + kStB, 0), dXmn0 = desc_mnmajor(st0 + kStX, 0);
            const uint64_t dHB = desc_mnmajor(smem_u32(sHB), 0), dWX = desc_mnmajor(smem_u32(sWX), 0);
            constexpr uint64_t kStageStep = (uint64_t)(kStageBytes >> 4);
            auto kstep_k = [](int k) -> uint64_t { return (uint64_t)(((k >> 2) * kTileHalf + (k & 3) * 32u) >> 4); };
            auto kstep_mn = [](int k) -> uint64_t { return (uint64_t)((k * 2048u) >> 4); };
            auto wait_ld = [&](int idx) {
                mbar_wait_bounded(bar_ld + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
            };
            auto mma_G = [&](int idx) {   // G = C B^T
                const uint64_t so = (idx & 1) ? kStageStep : 0;
                const uint64_t dC = dCk0 + so, dB = dBk0 + so;
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_bf16(tmem + kColG, dC + kstep_k(k), dB + kstep_k(k), kIdG, k > 0);
                umma_commit(bar_m1);
            };

            // A state-only item (long chains) runs only the state product,
            // the first of them without accumulating; the commits stay, so
            // every barrier keeps its phase.
            auto next_G = [&](int idx) {
                wait_ld(idx);
                tc_fence_after_sync();
                if (kLong && rg.is_pre(idx)) umma_commit(bar_m1);
                else mma_G(idx);
            };
            next_G(0);
            for (int idx = 0; idx < rg.count; ++idx) {
                const uint32_t ph = (uint32_t)idx & 1u;
                const uint64_t so = (idx & 1) ? kStageStep : 0;
                const uint64_t dC = dCk0 + so, dBmn = dBmn0 + so, dXmn = dXmn0 + so;
                const bool pre = kLong && rg.is_pre(idx);
                const uint32_t acc0 = pre && idx == rg.pre_begin() ? 0u : 1u;
                mbar_wait_bounded(bar_sready, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                if (!pre) {
                    const uint32_t dYo = tmem + kColYo + (uint32_t)(idx & 1) * 64u;
#pragma unroll
                    for (int k = 0; k < 8; ++k)   // Yo = C h^T
                        umma_bf16(dYo, dC + kstep_k(k), dHB + kstep_mn(k), kIdYo, k > 0);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)   // h += B^T (w o X)   (h already decayed)
                    umma_bf16(tmem + kColH, dBmn + kstep_mn(k), dWX + kstep_mn(k), kIdS, k > 0 ? 1u : acc0);
                umma_commit(bar_m4 + (idx & 1));
                mbar_wait_bounded(bar_mready, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                if (!pre) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)   // Yd = M X, M from TMEM
                        umma_bf16_tmem_a(tmem + kColYd, tmem + kColM + (uint32_t)k * 8u, dXmn + kstep_mn(k), kIdYd,
                                         k > 0);
                }
                umma_commit(bar_m2);
                if (idx + 1 < rg.count) next_G(idx + 1);   // the next item's C B^T (G was read: mready)
            }
        }
        __syncwarp();
    } else if (warp == kProdWarp) {
        // ------------------------------------------------------------------
        // producer warp (one thread): TMA loads, L2 prefetches and y stores
        // ------------------------------------------------------------------
        if (lane == 0 && rg.count > 0) {
            // The coordinates of an item, computed once (for its L2
            // prefetch) and passed along a rotation of items idx .. idx + 3.
            struct Co {
                int g, h, tok0, bi, nvalid;
                bool direct_y, pre;
            };
            int hint = rg.sB0;   // items are visited in increasing order
            auto coord = [&](int idx) {
                Co c{0, 0, 0, 0, 0, false, false};
                if (idx < rg.count) {
                    const Item it = item_at<kRagged, kLong>(prm, tabs, rg, idx, hint);
                    c = Co{group_of(it), it.h, it.tok0, it.bi, it.nvalid, it.direct_y, kLong && it.pre};
                }
                return c;
            };
            // B and C of item idx into its stage (G = C B^T needs only these;
            // a state-only item needs B alone)
            auto issue_bc = [&](int idx, const Co& c) {
                uint8_t* st = stage(idx);
                uint64_t* bar = bar_ld + (idx & 1);
                mbar_arrive_expect_tx(bar, kLong && c.pre ? kBytesBC / 2 : kBytesBC);
                tma_load_3d(st + kStB, &tmB, c.g * kN, c.tok0, c.bi, bar);
                tma_load_3d(st + kStB + kTileHalf, &tmB, c.g * kN + 64, c.tok0, c.bi, bar);
                if (!(kLong && c.pre)) {
                    tma_load_3d(st + kStC, &tmC, c.g * kN, c.tok0, c.bi, bar);
                    tma_load_3d(st + kStC + kTileHalf, &tmC, c.g * kN + 64, c.tok0, c.bi, bar);
                }
            };
            // X of item idx into its stage (the buffer that held y of item idx - 2)
            auto issue_x = [&](int idx, const Co& c) {
                uint64_t* bar = bar_ldx + (idx & 1);
                mbar_arrive_expect_tx(bar, kBytesX);
                tma_load_3d(stage(idx) + kStX, &tmX, c.h * kP, c.tok0, c.bi, bar);
            };
            // (long chains: the heads of a group walk the same chunks in step,
            // so B and C come from L2 and only X is prefetched; the B and C
            // prefetches there cost more TMA issue time than they save:
            // 2.66 -> 2.49 ms on 1 x 262144 tokens, 64 heads)
            auto prefetch_l2 = [&](const Co& c) {
                if constexpr (kLong) {
                    tma_prefetch_l2_3d(&tmX, c.h * kP, c.tok0, c.bi);
                    return;
                }
                tma_prefetch_l2_3d(&tmB, c.g * kN, c.tok0, c.bi);
                tma_prefetch_l2_3d(&tmB, c.g * kN + 64, c.tok0, c.bi);
                if (!(kLong && c.pre)) {
                    tma_prefetch_l2_3d(&tmC, c.g * kN, c.tok0, c.bi);
                    tma_prefetch_l2_3d(&tmC, c.g * kN + 64, c.tok0, c.bi);
                }
                tma_prefetch_l2_3d(&tmX, c.h * kP, c.tok0, c.bi);
            };
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmC);
            prefetch_tensormap(&tmY);
            Co c0 = coord(0), c1 = coord(1), c2 = coord(2), c3 = coord(3);   // items idx .. idx + 3
            issue_bc(0, c0);
            issue_x(0, c0);
            if (rg.count > 1) {
                issue_bc(1, c1);
                issue_x(1, c1);
            }
            if (rg.count > 2) prefetch_l2(c2);
            for (int idx = 0; idx < rg.count; ++idx) {
                const uint32_t sph = (uint32_t)(idx >> 1) & 1u;   // per-stage barrier parity
                // the state update, the last MMA reading B and C of item idx, is done
                mbar_wait_bounded(bar_m4 + (idx & 1), sph, kWaitNs, aborted, prm.status);
                if (idx + 2 < rg.count) issue_bc(idx + 2, c2);
                // y of item idx is staged in its X buffer: store it, then
                // reload the buffer once the store has read it
                mbar_wait_bounded(bar_ystaged + (idx & 1), sph, kWaitNs, aborted, prm.status);
                if (!(kLong && c0.pre)) {   // (a state-only item has no y)
                    if (!c0.direct_y) {
                        tma_store_3d(&tmY, stage(idx) + kStX, c0.h * kP, c0.tok0, c0.bi);
                    } else if constexpr (kRagged) {
                        // a partial last chunk: its rows up to the last
                        // multiple of 8 in boxes of 64, 32, 16, 8 rows (each
                        // starting on a whole swizzle atom); the rest went
                        // out row by row from the elementwise warps
                        const int nfull = c0.nvalid & ~7;
                        int off = 0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int rows = 64 >> q;
                            if (nfull & rows) {
                                tma_store_3d(&ypart.m[q], stage(idx) + kStX + off * 128, c0.h * kP, c0.tok0 + off,
                                             c0.bi);
                                off += rows;
                            }
                        }
                    }
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                if (idx + 2 < rg.count) issue_x(idx + 2, c2);
                if (idx + 3 < rg.count) prefetch_l2(c3);
                c0 = c1;
                c1 = c2;
                c2 = c3;
                c3 = coord(idx + 4);
            }
            bulk_wait_group0();   // all y stores complete before the CTA exits
        }
        __syncwarp();
    } else if (warp == kVecWarp) {
        // ------------------------------------------------------------------
        // vector warp: dt, cumulative decay and the off-diagonal column
        // factors of each chunk, published one chunk ahead.  The strided dt
        // loads of item idx + 1 are issued before item idx is computed, so
        // their latency is hidden behind a whole chunk.
        // ------------------------------------------------------------------
        struct DtIn {
            float a2, bias;
            int nvalid;   // tokens 4*lane + k with k < nvalid lie inside the sequence
            bool pre, pre_first;
            __nv_bfloat16 dt[4];
        };
        // raw inputs of item idx for tokens 4*lane .. 4*lane+3
        int hint = rg.sB0;
        auto load_dt = [&](int idx) {
            DtIn in;
            const Item it = item_at<kRagged, kLong>(prm, tabs, rg, idx, hint);
            in.a2 = prm.A[it.h] * 1.4426950408889634f;   // A * log2(e)
            in.bias = prm.dt_bias ? prm.dt_bias[it.h] : 0.0f;
            const __nv_bfloat16* dp = prm.dt_raw + ((size_t)it.bi * L + it.tok0 + lane * 4) * H + it.h;
            in.nvalid = it.nvalid - lane * 4;
            in.pre = it.pre;
            in.pre_first = it.pre_first;
#pragma unroll
            for (int k = 0; k < 4; ++k) in.dt[k] = k < in.nvalid ? dp[(size_t)k * H] : __float2bfloat16_rn(0.0f);
            return in;
        };
        // dt (0 past the sequence end), the inclusive cumulative log2 decay
        // (local sums, then a warp scan) and the off-diagonal column factor
        // 2^(cl_e - cl) dt, e the last token of the 32-token block.
        // A state-only item publishes instead, in the dt slot, its weights
        // w'_j = 2^(lrun + cl_last - cl_j) dt_j, lrun the log2 decay over the
        // chunks between it and the rebuilt state (walked back from there),
        // and in the v slot lrun including its own chunk.
        float vcl[4], vdt[4], vv[4];
        float lrun = 0.0f;
        auto compute_vecs = [&](const DtIn& in) {
            float run = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                vdt[k] = k < in.nvalid ? softplus_fast(__bfloat162float(in.dt[k]) + in.bias) : 0.0f;
                run += vdt[k] * in.a2;
                vcl[k] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const float excl = incl - run;
#pragma unroll
            for (int k = 0; k < 4; ++k) vcl[k] += excl;
            if (kLong && in.pre) {
                if (in.pre_first) lrun = 0.0f;
                const float cl_last = __shfl_sync(0xffffffffu, vcl[3], 31);
#pragma unroll
                for (int k = 0; k < 4; ++k) vdt[k] = ex2_approx(lrun + cl_last - vcl[k]) * vdt[k];
                lrun += cl_last;
#pragma unroll
                for (int k = 0; k < 4; ++k) vv[k] = lrun;
                return;
            }
            const float cl_e = __shfl_sync(0xffffffffu, vcl[3], lane | 7);
#pragma unroll
            for (int k = 0; k < 4; ++k) vv[k] = ex2_approx(cl_e - vcl[k]) * vdt[k];
        };
        auto publish_vecs = [&](int idx) {
            const ChunkVecs cv = chunk_vecs(smem, idx & 1);
            reinterpret_cast<float4*>(cv.cl)[lane] = make_float4(vcl[0], vcl[1], vcl[2], vcl[3]);
            reinterpret_cast<float4*>(cv.dt)[lane] = make_float4(vdt[0], vdt[1], vdt[2], vdt[3]);
            reinterpret_cast<float4*>(cv.v)[lane] = make_float4(vv[0], vv[1], vv[2], vv[3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_vec);
        };

        if (rg.count > 0) {
            DtIn in = load_dt(0);
            compute_vecs(in);
            publish_vecs(0);
            if (rg.count > 1) {
                in = load_dt(1);
                compute_vecs(in);
            }
            if (rg.count > 2) in = load_dt(2);
            for (int idx = 0; idx + 1 < rg.count; ++idx) {
                // The elementwise warps waited for vectors idx before arriving
                // for item idx's state products, and read vectors idx - 1 only
                // before the masked tile of item idx - 1 was ready (earlier
                // still), so buffer (idx + 1) & 1 is free.
                if (lane == 0) mbar_wait_bounded(bar_sready, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                __syncwarp();
                publish_vecs(idx + 1);
                if (idx + 2 < rg.count) {
                    compute_vecs(in);
                    if (idx + 3 < rg.count) in = load_dt(idx + 3);
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------
        // elementwise warps
        // ------------------------------------------------------------------
        const int quad = warp & 3;          // TMEM lane quadrant
        const int quarter = warp >> 2;      // column quarter
        const int row = quad * 32 + lane;   // token row i / state column n
        const int p0 = quarter * 16;        // this thread's 16 columns p
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tH = tmem + kColH + (uint32_t)p0 + lane_off;

        // the initial state of chain ch's sequence and head (16 columns p of
        // state column n = row), or zeros
        auto load_init = [&](int ch, float (&hv)[16]) {
            const float* src = prm.init_state ? prm.init_state + (size_t)ch * (kP * kN) : nullptr;
#pragma unroll
            for (int p = 0; p < 16; ++p) hv[p] = src ? src[(size_t)(p0 + p) * kN + row] : 0.0f;
        };
        // the state published by the predecessor CTA (bounded wait on its
        // flag).  The ranges of a long-memory chain publish one after
        // another, so the bound allows for the chain's chunks before this
        // range as well.
        auto load_published = [&](float (&hv)[16]) {
            const int* flag = prm.ws_ctrl + 16 + (ticket - 1);
            const uint64_t limit = kWaitNs + (uint64_t)rg.startC * kWaitPerChunkNs;
            if (tid == 0 && !*aborted) {
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(flag) == 0) {
                    if (globaltimer_ns() - t0 > limit) {
                        *aborted = 1;
                        if (prm.status) atomicExch(reinterpret_cast<int*>(prm.status), 4);
                        break;
                    }
                }
            }
            named_bar_sync(kEwBarrier, kEwThreads);
            const float* src = prm.ws_states + (size_t)(ticket - 1) * (kP * kN);
#pragma unroll
            for (int p = 0; p < 16; ++p) hv[p] = __ldcg(src + (size_t)(p0 + p) * kN + row);
        };
        // the state-only items (long chains) left a valid starting state in
        // the TMEM state columns
        bool pre_ok = false;

        // state entering a segment: the initial state, the rebuilt state,
        // the predecessor CTA's published state (a dependent segment), or zero
        auto segment_state = [&](const Item& it, float (&hv)[16]) {
            if (it.depend) {
                if (kLong && pre_ok) {
                    tmem_ld16(tH, hv);
                    tmem_wait_ld();
                } else {
                    load_published(hv);
                }
            } else {
                load_init(it.chain, hv);
            }
        };

        // y of item j = Yd + 2^cl Yo (token row `row`, this quarter's p; D x
        // is in Yd through M's diagonal), written over x in the item's X
        // buffer for the producer's TMA store.  M X of item j (the X
        // buffer's last reader) is done once bar_m2 has completed for it.
        // A state-only item has no y: its barriers are still passed.
        // the previous item's row placement (ragged batches only)
        int prev_tok0 = 0, prev_nvalid = 0, prev_h = 0;
        bool prev_direct = false, prev_pre = false;
        auto y_epilogue = [&](int j, float cl_i) {
            mbar_wait_bounded(bar_m2, (uint32_t)j & 1u, kWaitNs, aborted, prm.status);
            if (kLong && prev_pre) {
                mbar_arrive(bar_ystaged + (j & 1));
                return;
            }
            tc_fence_after_sync();
            uint8_t* xs = stage(j) + kStX;
            const float sc = ex2_approx(cl_i);
            float yd[16], yo[16];
            tmem_ld16(tmem + kColYd + lane_off + (uint32_t)p0, yd);
            tmem_ld16(tmem + kColYo + (uint32_t)(j & 1) * 64u + lane_off + (uint32_t)p0, yo);
            tmem_wait_ld();
            uint4 packed[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float2 r = fma2(make_float2(sc, sc), make_float2(yo[q * 8 + e], yo[q * 8 + e + 1]),
                                          make_float2(yd[q * 8 + e], yd[q * 8 + e + 1]));
                    o[e] = r.x;
                    o[e + 1] = r.y;
                }
                packed[q] = pack_bf16x8(o);
            }
            if constexpr (kRagged) {
                // a ragged batch's partial last chunk: its rows past the
                // sequence's end belong to the next sequence, so no 128-row
                // box goes out; the producer stores the rows up to the last
                // multiple of 8 in smaller boxes, and the rest go out here
                if (prev_direct && row >= (prev_nvalid & ~7) && row < prev_nvalid) {
                    __nv_bfloat16* yr = prm.y + ((size_t)(prev_tok0 + row) * H + prev_h) * kP + p0;
                    reinterpret_cast<uint4*>(yr)[0] = packed[0];
                    reinterpret_cast<uint4*>(yr)[1] = packed[1];
                }
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) *reinterpret_cast<uint4*>(xs + sw128(row, quarter * 2 + q)) = packed[q];
            fence_proxy_async_smem();
            mbar_arrive(bar_ystaged + (j & 1));
        };

        float prev_cl_i = 0.0f;
        int hint = rg.sB0;
        for (int idx = 0; idx < rg.count; ++idx) {
            const Item it = item_at<kRagged, kLong>(prm, tabs, rg, idx, hint);
            const int bi = it.seq, h = it.h;
            uint8_t* st = stage(idx);
            float cl_i = 0.0f;

            if (kLong && it.pre) {
                // ----------------------------------------------------------
                // state-only item: w' o X for S += B^T (w' o X), no state
                // carried in TMEM between these items (the MMAs accumulate)
                // ----------------------------------------------------------
                mbar_wait_bounded(bar_vec, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                const ChunkVecs cv = chunk_vecs(smem, idx & 1);
                const float wj = cv.dt[row];
                const float lsum = cv.v[0];   // log2 decay from this chunk's start to the rebuilt state
                // the previous item's state product, which reads the w o X
                // buffer, is done
                if (idx > 0)
                    mbar_wait_bounded(bar_m4 + ((idx - 1) & 1), (uint32_t)((idx - 1) >> 1) & 1u, kWaitNs, aborted,
                                      prm.status);
                mbar_wait_bounded(bar_ldx + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
                const __nv_bfloat162 w2 = __floats2bfloat162_rn(wj, wj);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    *reinterpret_cast<uint4*>(sWX + sw128(row, quarter * 2 + q)) =
                        scale_bf16x8(*reinterpret_cast<const uint4*>(st + kStX + sw128(row, quarter * 2 + q)), w2);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(bar_sready);   // the state product can start
                if (idx > 0) y_epilogue(idx - 1, prev_cl_i);
                mbar_wait_bounded(bar_m1, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                tc_fence_before_sync();
                mbar_arrive(bar_mready);   // (no masked tile)
                if (it.pre_last) {
                    // the walk is over: the rebuilt state is exact when it
                    // reached the chain's start (plus the decayed initial
                    // state), or when the accumulated decay is below 2^-64
                    // (the last state product is waited for either way: the
                    // next item rewrites the state columns)
                    const bool from_start = rg.startC - rg.npre == 0;
                    pre_ok = from_start || lsum <= kPreCutLog2;
                    mbar_wait_bounded(bar_m4 + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
                    tc_fence_after_sync();
                    if (from_start && prm.init_state) {
                        float hs[16], h0[16];
                        tmem_ld16(tH, hs);
                        load_init(it.chain, h0);
                        tmem_wait_ld();
                        const float d0 = ex2_approx(lsum);
#pragma unroll
                        for (int p = 0; p < 16; ++p) hs[p] = fmaf(d0, h0[p], hs[p]);
                        tmem_st16(tH, hs);
                        tmem_wait_st();
                    }
                }
                prev_pre = true;
                prev_cl_i = 0.0f;
                continue;
            }

            const float Dh = prm.D ? prm.D[h] : 0.0f;
            // 1. the state entering item idx (fp32, state column n = row)
            float hv[16];
            if (it.seg_start) {
                segment_state(it, hv);
            } else {
                // the previous item's C h^T and state update are done, so
                // the state, its bf16 copy and w o X buffers are free
                mbar_wait_bounded(bar_m4 + ((idx - 1) & 1), (uint32_t)((idx - 1) >> 1) & 1u, kWaitNs, aborted,
                                  prm.status);
                tc_fence_after_sync();
                tmem_ld16(tH, hv);
                tmem_wait_ld();
            }
            // 2. its bf16 copy for C h^T
#pragma unroll
            for (int q = 0; q < 2; ++q)
                *reinterpret_cast<uint4*>(sHB + sw128(row, (p0 >> 3) + q)) = pack_bf16x8(&hv[q * 8]);

            // 3. the decayed state back into TMEM (the state product
            //    accumulates onto it) and w o X, w_j = 2^(cl_last - cl_j) dt_j
            mbar_wait_bounded(bar_vec, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
            const ChunkVecs cv = chunk_vecs(smem, idx & 1);
            cl_i = cv.cl[row];
            const float cl_last = cv.cl[kQ - 1];
            {
                const float decay = ex2_approx(cl_last);
#pragma unroll
                for (int p = 0; p < 16; p += 2) {
                    const float2 r = mul2(make_float2(hv[p], hv[p + 1]), make_float2(decay, decay));
                    hv[p] = r.x;
                    hv[p + 1] = r.y;
                }
                tmem_st16(tH, hv);
            }
            mbar_wait_bounded(bar_ldx + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
            {
                const float wj = ex2_approx(cl_last - cl_i) * cv.dt[row];
                const __nv_bfloat162 w2 = __floats2bfloat162_rn(wj, wj);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    *reinterpret_cast<uint4*>(sWX + sw128(row, quarter * 2 + q)) =
                        scale_bf16x8(*reinterpret_cast<const uint4*>(st + kStX + sw128(row, quarter * 2 + q)), w2);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_sready);   // C h^T and the state update can start

            // 4. y of the previous item, whose M X ran meanwhile
            if (idx > 0) y_epilogue(idx - 1, prev_cl_i);

            // 5. the masked tile M = G o L of item idx into TMEM (bf16
            //    pairs), the A operand of M X.  Column block jb (32 tokens)
            //    is zero above the row quadrant's diagonal block; of every
            //    block, column quarter `quarter` takes 8 columns.  One block
            //    at a time, in a loop that is not unrolled: the smaller code
            //    is faster (3B layer 0.0963 -> 0.0943 ms).
            mbar_wait_bounded(bar_m1, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            {
#pragma unroll 1
                for (int jb = 0; jb < 4; ++jb) {
                    const int j0 = jb * 32 + quarter * 8;
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    float gb[8];
                    if (jb <= quad) {
                        tmem_ld8(tmem + kColG + lane_off + (uint32_t)j0, gb);
                        tmem_wait_ld();
                    }
                    if (jb < quad) {
                        const float u = ex2_approx(cl_i - cv.cl[jb * 32 + 31]);
                        const float4 va = reinterpret_cast<const float4*>(cv.v + j0)[0];
                        const float4 vb = reinterpret_cast<const float4*>(cv.v + j0)[1];
                        const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 uv = mul2(make_float2(u, u), make_float2(vv[2 * e], vv[2 * e + 1]));
                            const float2 m = mul2(make_float2(gb[2 * e], gb[2 * e + 1]), uv);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(m.x, m.y);
                            w[e] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                    } else if (jb == quad) {
                        const float4 ca = reinterpret_cast<const float4*>(cv.cl + j0)[0];
                        const float4 cb = reinterpret_cast<const float4*>(cv.cl + j0)[1];
                        const float4 da = reinterpret_cast<const float4*>(cv.dt + j0)[0];
                        const float4 db = reinterpret_cast<const float4*>(cv.dt + j0)[1];
                        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                        const float dd[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
                        // diagonal element: + D (so that M X includes D x)
                        float m[8];
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 f = mul2(make_float2(ex2_approx(cl_i - cc[e]), ex2_approx(cl_i - cc[e + 1])),
                                                  make_float2(dd[e], dd[e + 1]));
                            const float2 v = mul2(make_float2(gb[e], gb[e + 1]), f);
                            m[e] = (j0 + e < row) ? v.x : (j0 + e == row ? v.x + Dh : 0.0f);
                            m[e + 1] = (j0 + e + 1 < row) ? v.y : (j0 + e + 1 == row ? v.y + Dh : 0.0f);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(m[2 * e], m[2 * e + 1]);
                            w[e] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                    }
                    tmem_st4(tmem + kColM + lane_off + (uint32_t)(j0 >> 1), w[0], w[1], w[2], w[3]);
                }
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_mready);   // M X can start

            // 6. end of a segment: the state leaves the chip
            if (it.seg_end) {
                mbar_wait_bounded(bar_m4 + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                tmem_ld16(tH, hv);
                tmem_wait_ld();
                if (it.publish) {
                    float* dst = prm.ws_states + (size_t)ticket * (kP * kN);
#pragma unroll
                    for (int p = 0; p < 16; ++p) __stcg(dst + (size_t)(p0 + p) * kN + row, hv[p]);
                    __threadfence();
                    named_bar_sync(kEwBarrier, kEwThreads);
                    if (tid == 0) st_release_gpu(prm.ws_ctrl + 16 + ticket, 1);
                } else if (prm.final_state) {
                    float* dst = prm.final_state + ((size_t)bi * H + h) * (size_t)(kP * kN);
#pragma unroll
                    for (int p = 0; p < 16; ++p) dst[(size_t)(p0 + p) * kN + row] = hv[p];
                }
            }
            prev_cl_i = cl_i;
            prev_pre = false;
            if constexpr (kRagged) {
                prev_tok0 = it.tok0;
                prev_nvalid = it.nvalid;
                prev_h = it.h;
                prev_direct = it.direct_y;
            }
        }
        if (rg.count > 0) y_epilogue(rg.count - 1, prev_cl_i);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Head pairs.  When a group has an even number of heads, an item is two
// heads h, h + 1 of one group over one chunk.  They share B, C and G, so B
// and C are loaded and C B^T computed once per pair, and their states sit
// side by side in TMEM (lane n, columns [h p | h+1 p]), so that both state
// products are one N = 128 MMA chain and so are both C h^T.  The elementwise
// warps run one chain of steps per pair rather than one per head.
//   TMEM: G [0,128); M of the two heads [128,256) (bf16 pairs); Y of the two
//   heads [256,384): C h^T, scaled in place by 2^(cl_i) by the elementwise
//   warps, then M X accumulated onto it, so Y = y; the state pair [384,512).
//   Shared memory: one B/C buffer, reloaded once the item's last product
//   reading it (C h^T) is done; two X stages holding both heads' tiles, over
//   which y is staged; the bf16 state pair; w o X of both heads.
// Per item the MMA warp issues the state product once the state is
// released, C h^T once the previous item's y has been read from TMEM, both
// heads' M X once the masked tiles and the scaled C h^T are in TMEM, then
// the next item's G.  The elementwise warps release the state, read the
// previous y, build both masked tiles from one read of G and scale C h^T.
// Elementwise warp w serves TMEM lanes 32*(w%4).. and column quarter w/4:
// for the state, w o X and y, quarter q is head q/2, columns p of
// 32*(q%2)..; for the masked tiles, 8 columns of every 32-token block, for
// both heads.
// ---------------------------------------------------------------------------
namespace pr {
constexpr int kStB = 0, kStC = 32768;       // the B/C buffer, two 16 KB halves each
constexpr int kOffX = 65536;                 // two X stages [128 tok][h p | h+1 p]
constexpr int kXStage = 32768;
constexpr int kOffHB = kOffX + 2 * kXStage;  // bf16 state pair [128 n][h p | h+1 p]
constexpr int kOffWX = kOffHB + 32768;       // w o X of both heads [128 tok][h p | h+1 p]
constexpr int kOffVec = kOffWX + 32768;      // per parity and head: cl, dt, v (float[128] each)
constexpr int kVecHead = 3 * kQ, kVecSet = 2 * kVecHead;
constexpr int kOffBar = kOffVec + 2 * kVecSet * 4;
constexpr int kNumBars = 13;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr uint32_t kColG = 0, kColM = 128, kColY = 256, kColH = 384;
constexpr uint32_t kIdYo = umma_idesc_bf16(128, 128, false, true);   // C (K-maj) x state pair (MN-maj)
constexpr uint32_t kIdS = umma_idesc_bf16(128, 128, true, true);     // B^T (MN-maj) x (w o X) pair (MN-maj)
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace pr

// 32 TMEM columns of a lane as two 16-column accesses: in the pair kernel
// this is 2% faster on the 8B layer than one 32-column access and gives the
// same values (the register allocator places two short vectors more freely).
__device__ inline void pair_ld32(uint32_t taddr, float (&v)[32])
{
    float a[16], b[16];
    tmem_ld16(taddr, a);
    tmem_ld16(taddr + 16u, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[i] = a[i];
        v[16 + i] = b[i];
    }
}
__device__ inline void pair_st32(uint32_t taddr, const float (&v)[32])
{
    float a[16], b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = v[i];
        b[i] = v[16 + i];
    }
    tmem_st16(taddr, a);
    tmem_st16(taddr + 16u, b);
}

template <bool kLong>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
                          const __grid_constant__ YBoxes ypart, const Params prm)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pr::kOffBar);
    uint64_t* bar_ld = bars + 0;        // B (and C) landed in the B/C buffer (TMA)
    uint64_t* bar_ldx = bars + 1;       // [2]: stage's X landed (TMA)
    uint64_t* bar_vec = bars + 3;       // chunk vectors published (vector warp)
    uint64_t* bar_sready = bars + 4;    // bf16 state, w o X and decayed state ready (elementwise warps)
    uint64_t* bar_m4 = bars + 5;        // state product done
    uint64_t* bar_yread = bars + 6;     // previous item's y read from TMEM (elementwise warps)
    uint64_t* bar_myo = bars + 7;       // C h^T done, and every earlier product: the B/C buffer is free
    uint64_t* bar_m1 = bars + 8;        // G done
    uint64_t* bar_mready = bars + 9;    // masked tiles and scaled C h^T in TMEM; G read (elementwise warps)
    uint64_t* bar_m2 = bars + 10;       // M X done: y in TMEM
    uint64_t* bar_ystaged = bars + 11;  // [2]: y staged in the stage's X buffer (elementwise warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + pr::kOffMisc);
    volatile int* aborted = reinterpret_cast<volatile int*>(smem + pr::kOffMisc + 4);
    int* ticket_slot = reinterpret_cast<int*>(smem + pr::kOffMisc + 8);
    const int L = prm.L, Hf = prm.Hf;

    if (tid == 0) {
        *aborted = 0;
        mbar_init(bar_ld, 1);
        mbar_init(bar_ldx, 1);
        mbar_init(bar_ldx + 1, 1);
        mbar_init(bar_vec, 1);
        mbar_init(bar_sready, kEwThreads);
        mbar_init(bar_m4, 1);
        mbar_init(bar_yread, kEwThreads);
        mbar_init(bar_myo, 1);
        mbar_init(bar_m1, 1);
        mbar_init(bar_mready, kEwThreads);
        mbar_init(bar_m2, 1);
        mbar_init(bar_ystaged, kEwThreads);
        mbar_init(bar_ystaged + 1, kEwThreads);
        fence_mbar_init();
        *ticket_slot = atomicAdd(prm.ws_ctrl, 1);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int ticket = *ticket_slot;
    const Tabs tabs{nullptr, nullptr, nullptr};
    const Range rg = make_range<false, kLong>(prm, tabs, ticket, prm.units);
    auto group_of = [&](const Item& it) { return (int)prm.fHG.div((uint32_t)it.h); };
    auto xstage = [&](int idx) { return smem + pr::kOffX + (idx & 1) * pr::kXStage; };
    // per parity and head: cl, dt, v
    auto vecs = [&](int parity, int hd) {
        return reinterpret_cast<float*>(smem + pr::kOffVec) + parity * pr::kVecSet + hd * pr::kVecHead;
    };

    if (warp == kMmaWarp) {
        // ------------------------------------------------------------------
        // MMA warp (one thread)
        // ------------------------------------------------------------------
        if (lane == 0 && rg.count > 0) {
            const uint32_t sbc = smem_u32(smem);
            const uint64_t dCk = desc_kmajor(sbc + pr::kStC, 0), dBk = desc_kmajor(sbc + pr::kStB, 0);
            const uint64_t dBmn = desc_mnmajor(sbc + pr::kStB, 0);
            const uint64_t dHB = desc_mnmajor(smem_u32(smem + pr::kOffHB), 0);
            const uint64_t dWX = desc_mnmajor(smem_u32(smem + pr::kOffWX), 0);
            const uint64_t dX0 = desc_mnmajor(smem_u32(smem + pr::kOffX), 0);
            constexpr uint64_t kXStep = (uint64_t)(pr::kXStage >> 4), kHalfStep = (uint64_t)(kTileHalf >> 4);
            auto kstep_k = [](int k) -> uint64_t { return (uint64_t)(((k >> 2) * kTileHalf + (k & 3) * 32u) >> 4); };
            auto kstep_mn = [](int k) -> uint64_t { return (uint64_t)((k * 2048u) >> 4); };
            // G = C B^T of item idx (a state-only item has none; the commit stays)
            auto next_G = [&](int idx) {
                mbar_wait_bounded(bar_ld, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                if (!(kLong && rg.is_pre(idx))) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        umma_bf16(tmem + pr::kColG, dCk + kstep_k(k), dBk + kstep_k(k), kIdG, k > 0);
                }
                umma_commit(bar_m1);
            };
            next_G(0);
            for (int idx = 0; idx < rg.count; ++idx) {
                const uint32_t ph = (uint32_t)idx & 1u;
                const bool pre = kLong && rg.is_pre(idx);
                const uint32_t acc0 = pre && idx == rg.pre_begin() ? 0u : 1u;
                mbar_wait_bounded(bar_sready, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)   // [h | h+1] += B^T (w o X)   (the states already decayed)
                    umma_bf16(tmem + pr::kColH, dBmn + kstep_mn(k), dWX + kstep_mn(k), pr::kIdS, k > 0 ? 1u : acc0);
                umma_commit(bar_m4);
                mbar_wait_bounded(bar_yread, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                if (!pre) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)   // Y = C [h | h+1]^T
                        umma_bf16(tmem + pr::kColY, dCk + kstep_k(k), dHB + kstep_mn(k), pr::kIdYo, k > 0);
                }
                umma_commit(bar_myo);
                mbar_wait_bounded(bar_mready, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                if (!pre) {
                    const uint64_t dX = dX0 + (idx & 1) * kXStep;
#pragma unroll
                    for (int hd = 0; hd < 2; ++hd)
#pragma unroll
                        for (int k = 0; k < 8; ++k)   // Y += M X, per head (M from TMEM)
                            umma_bf16_tmem_a(tmem + pr::kColY + (uint32_t)hd * 64u,
                                             tmem + pr::kColM + (uint32_t)hd * 64u + (uint32_t)k * 8u,
                                             dX + (uint64_t)hd * kHalfStep + kstep_mn(k), kIdYd, 1u);
                }
                umma_commit(bar_m2);
                if (idx + 1 < rg.count) next_G(idx + 1);
            }
        }
        __syncwarp();
    } else if (warp == kProdWarp) {
        // ------------------------------------------------------------------
        // producer warp (one thread)
        // ------------------------------------------------------------------
        if (lane == 0 && rg.count > 0) {
            struct Co {
                int g, h, tok0, bi;   // h: the pair's first head
                bool pre;
            };
            int hint = rg.sB0;
            auto coord = [&](int idx) {
                Co c{0, 0, 0, 0, false};
                if (idx < rg.count) {
                    const Item it = item_at<false, kLong>(prm, tabs, rg, idx, hint);
                    c = Co{group_of(it), 2 * it.h, it.tok0, it.bi, kLong && it.pre};
                }
                return c;
            };
            auto issue_bc = [&](const Co& c) {
                mbar_arrive_expect_tx(bar_ld, c.pre ? kBytesBC / 2 : kBytesBC);
                tma_load_3d(smem + pr::kStB, &tmB, c.g * kN, c.tok0, c.bi, bar_ld);
                tma_load_3d(smem + pr::kStB + kTileHalf, &tmB, c.g * kN + 64, c.tok0, c.bi, bar_ld);
                if (!c.pre) {
                    tma_load_3d(smem + pr::kStC, &tmC, c.g * kN, c.tok0, c.bi, bar_ld);
                    tma_load_3d(smem + pr::kStC + kTileHalf, &tmC, c.g * kN + 64, c.tok0, c.bi, bar_ld);
                }
            };
            auto issue_x = [&](int idx, const Co& c) {
                uint64_t* bar = bar_ldx + (idx & 1);
                mbar_arrive_expect_tx(bar, 2 * kBytesX);
                tma_load_3d(xstage(idx), &tmX, c.h * kP, c.tok0, c.bi, bar);
                tma_load_3d(xstage(idx) + kTileHalf, &tmX, c.h * kP + kP, c.tok0, c.bi, bar);
            };
            // (long chains: a group's pairs walk the same chunks in step, so
            // B and C come from L2 and only X is prefetched)
            auto prefetch_l2 = [&](const Co& c) {
                tma_prefetch_l2_3d(&tmX, c.h * kP, c.tok0, c.bi);
                tma_prefetch_l2_3d(&tmX, c.h * kP + kP, c.tok0, c.bi);
                if constexpr (!kLong) {
                    tma_prefetch_l2_3d(&tmB, c.g * kN, c.tok0, c.bi);
                    tma_prefetch_l2_3d(&tmB, c.g * kN + 64, c.tok0, c.bi);
                    tma_prefetch_l2_3d(&tmC, c.g * kN, c.tok0, c.bi);
                    tma_prefetch_l2_3d(&tmC, c.g * kN + 64, c.tok0, c.bi);
                }
            };
            prefetch_tensormap(&tmX);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmC);
            prefetch_tensormap(&tmY);
            Co c0 = coord(0), c1 = coord(1), c2 = coord(2), c3 = coord(3);   // items idx .. idx + 3
            issue_bc(c0);
            issue_x(0, c0);
            if (rg.count > 1) {
                issue_x(1, c1);
                prefetch_l2(c1);
            }
            if (rg.count > 2) prefetch_l2(c2);
            for (int idx = 0; idx < rg.count; ++idx) {
                const uint32_t sph = (uint32_t)(idx >> 1) & 1u;
                // C h^T of item idx, the last product reading B and C, is done
                mbar_wait_bounded(bar_myo, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                if (idx + 1 < rg.count) issue_bc(c1);
                // y of item idx is staged in its X stage: store it, then
                // reload the stage once the stores have read it
                mbar_wait_bounded(bar_ystaged + (idx & 1), sph, kWaitNs, aborted, prm.status);
                if (!c0.pre) {
                    tma_store_3d(&tmY, xstage(idx), c0.h * kP, c0.tok0, c0.bi);
                    tma_store_3d(&tmY, xstage(idx) + kTileHalf, c0.h * kP + kP, c0.tok0, c0.bi);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                if (idx + 2 < rg.count) issue_x(idx + 2, c2);
                if (idx + 3 < rg.count) prefetch_l2(c3);
                c0 = c1;
                c1 = c2;
                c2 = c3;
                c3 = coord(idx + 4);
            }
            bulk_wait_group0();
        }
        __syncwarp();
    } else if (warp == kVecWarp) {
        // ------------------------------------------------------------------
        // vector warp: both heads' dt, cumulative decay and off-diagonal
        // column factors (as in the one-head kernel), one chunk ahead
        // ------------------------------------------------------------------
        struct DtIn {
            float a2[2], bias[2];
            int nvalid;
            bool pre, pre_first;
            __nv_bfloat16 dt[2][4];
        };
        int hint = rg.sB0;
        auto load_dt = [&](int idx) {
            DtIn in;
            const Item it = item_at<false, kLong>(prm, tabs, rg, idx, hint);
            const int h0 = 2 * it.h;
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
                in.a2[hd] = prm.A[h0 + hd] * 1.4426950408889634f;
                in.bias[hd] = prm.dt_bias ? prm.dt_bias[h0 + hd] : 0.0f;
            }
            const __nv_bfloat16* dp = prm.dt_raw + ((size_t)it.bi * L + it.tok0 + lane * 4) * Hf + h0;
            in.nvalid = it.nvalid - lane * 4;
            in.pre = it.pre;
            in.pre_first = it.pre_first;
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int hd = 0; hd < 2; ++hd)
                    in.dt[hd][k] = k < in.nvalid ? dp[(size_t)k * Hf + hd] : __float2bfloat16_rn(0.0f);
            return in;
        };
        float vcl[2][4], vdt[2][4], vv[2][4];
        float lrun[2] = {0.0f, 0.0f};
        auto compute_vecs = [&](const DtIn& in) {
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
                float run = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    vdt[hd][k] = k < in.nvalid ? softplus_fast(__bfloat162float(in.dt[hd][k]) + in.bias[hd]) : 0.0f;
                    run += vdt[hd][k] * in.a2[hd];
                    vcl[hd][k] = run;
                }
                float incl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                const float excl = incl - run;
#pragma unroll
                for (int k = 0; k < 4; ++k) vcl[hd][k] += excl;
                if (kLong && in.pre) {
                    if (in.pre_first) lrun[hd] = 0.0f;
                    const float cl_last = __shfl_sync(0xffffffffu, vcl[hd][3], 31);
#pragma unroll
                    for (int k = 0; k < 4; ++k) vdt[hd][k] = ex2_approx(lrun[hd] + cl_last - vcl[hd][k]) * vdt[hd][k];
                    lrun[hd] += cl_last;
#pragma unroll
                    for (int k = 0; k < 4; ++k) vv[hd][k] = lrun[hd];
                    continue;
                }
                const float cl_e = __shfl_sync(0xffffffffu, vcl[hd][3], lane | 7);
#pragma unroll
                for (int k = 0; k < 4; ++k) vv[hd][k] = ex2_approx(cl_e - vcl[hd][k]) * vdt[hd][k];
            }
        };
        auto publish_vecs = [&](int idx) {
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
                float* b = vecs(idx & 1, hd);
                reinterpret_cast<float4*>(b)[lane] = make_float4(vcl[hd][0], vcl[hd][1], vcl[hd][2], vcl[hd][3]);
                reinterpret_cast<float4*>(b + kQ)[lane] = make_float4(vdt[hd][0], vdt[hd][1], vdt[hd][2], vdt[hd][3]);
                reinterpret_cast<float4*>(b + 2 * kQ)[lane] = make_float4(vv[hd][0], vv[hd][1], vv[hd][2], vv[hd][3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_vec);
        };
        if (rg.count > 0) {
            DtIn in = load_dt(0);
            compute_vecs(in);
            publish_vecs(0);
            if (rg.count > 1) {
                in = load_dt(1);
                compute_vecs(in);
            }
            if (rg.count > 2) in = load_dt(2);
            for (int idx = 0; idx + 1 < rg.count; ++idx) {
                // vectors idx - 1 were last read before the masked tiles of
                // item idx - 1 were ready, earlier than this item's release
                if (lane == 0) mbar_wait_bounded(bar_sready, (uint32_t)idx & 1u, kWaitNs, aborted, prm.status);
                __syncwarp();
                publish_vecs(idx + 1);
                if (idx + 2 < rg.count) {
                    compute_vecs(in);
                    if (idx + 3 < rg.count) in = load_dt(idx + 3);
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------
        // elementwise warps
        // ------------------------------------------------------------------
        const int quad = warp & 3;          // TMEM lane quadrant
        const int quarter = warp >> 2;      // column quarter
        const int row = quad * 32 + lane;   // token row i / state column n
        const int hd = quarter >> 1;        // this thread's head of the pair (state, w o X, y)
        const int pq = (quarter & 1) * 32;  // its 32 columns p of that head
        const int ch0 = pq >> 3;            // their first 16-byte chunk in a 128-byte row
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tH = tmem + pr::kColH + (uint32_t)(hd * 64 + pq) + lane_off;
        const uint32_t tY = tmem + pr::kColY + (uint32_t)(hd * 64 + pq) + lane_off;
        uint8_t* sHB = smem + pr::kOffHB + hd * kTileHalf;
        uint8_t* sWX = smem + pr::kOffWX + hd * kTileHalf;
        constexpr size_t kPN = (size_t)kP * kN;

        // the initial state of this thread's head of pair chain ch (32
        // columns p of state column n = row), or zeros
        auto load_init = [&](int ch, float (&hv)[32]) {
            const int seq = (int)prm.fH.div((uint32_t)ch);
            const int h = 2 * (ch - seq * prm.H) + hd;
            const float* src = prm.init_state ? prm.init_state + ((size_t)seq * Hf + h) * kPN : nullptr;
#pragma unroll
            for (int p = 0; p < 32; ++p) hv[p] = src ? src[(size_t)(pq + p) * kN + row] : 0.0f;
        };
        auto load_published = [&](float (&hv)[32]) {
            const int* flag = prm.ws_ctrl + 16 + (ticket - 1);
            const uint64_t limit = kWaitNs + (uint64_t)rg.startC * kWaitPerChunkNs;
            if (tid == 0 && !*aborted) {
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(flag) == 0) {
                    if (globaltimer_ns() - t0 > limit) {
                        *aborted = 1;
                        if (prm.status) atomicExch(reinterpret_cast<int*>(prm.status), 4);
                        break;
                    }
                }
            }
            named_bar_sync(kEwBarrier, kEwThreads);
            const float* src = prm.ws_states + ((size_t)(ticket - 1) * 2 + hd) * kPN;
#pragma unroll
            for (int p = 0; p < 32; ++p) hv[p] = __ldcg(src + (size_t)(pq + p) * kN + row);
        };
        bool pre_ok = false;
        auto segment_state = [&](const Item& it, float (&hv)[32]) {
            if (it.depend) {
                if (kLong && pre_ok) {
                    pair_ld32(tH, hv);
                    tmem_wait_ld();
                } else {
                    load_published(hv);
                }
            } else {
                load_init(it.chain, hv);
            }
        };
        // y of item j (Y, this thread's head and columns), staged over the
        // item's X tiles for the producer's TMA stores; then (unless it is
        // the last) the arrival that lets C h^T of the next item into Y
        bool prev_pre = false;
        auto y_epilogue = [&](int j, bool release) {
            mbar_wait_bounded(bar_m2, (uint32_t)j & 1u, kWaitNs, aborted, prm.status);
            if (kLong && prev_pre) {
                mbar_arrive(bar_ystaged + (j & 1));
                if (release) mbar_arrive(bar_yread);
                return;
            }
            tc_fence_after_sync();
            float yv[32];
            pair_ld32(tY, yv);
            tmem_wait_ld();
            if (release) {
                tc_fence_before_sync();
                mbar_arrive(bar_yread);
            }
            uint8_t* xs = xstage(j) + hd * kTileHalf;
#pragma unroll
            for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(xs + sw128(row, ch0 + q)) = pack_bf16x8(&yv[q * 8]);
            fence_proxy_async_smem();
            mbar_arrive(bar_ystaged + (j & 1));
        };

        int hint = rg.sB0;
        for (int idx = 0; idx < rg.count; ++idx) {
            const Item it = item_at<false, kLong>(prm, tabs, rg, idx, hint);
            const int h0 = 2 * it.h;
            const uint32_t ph = (uint32_t)idx & 1u;
            uint8_t* xs = xstage(idx) + hd * kTileHalf;
            const float* cv = vecs(idx & 1, hd);

            if (kLong && it.pre) {
                // ----------------------------------------------------------
                // state-only item: w' o X of both heads
                // ----------------------------------------------------------
                mbar_wait_bounded(bar_vec, ph, kWaitNs, aborted, prm.status);
                const float wj = cv[kQ + row];
                const float lsum = cv[2 * kQ];   // this head's log2 decay from the chunk's start to the rebuilt state
                const bool both_cut = vecs(idx & 1, 0)[2 * kQ] <= kPreCutLog2 && vecs(idx & 1, 1)[2 * kQ] <= kPreCutLog2;
                if (idx > 0)
                    mbar_wait_bounded(bar_m4, (uint32_t)(idx - 1) & 1u, kWaitNs, aborted, prm.status);
                mbar_wait_bounded(bar_ldx + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
                const __nv_bfloat162 w2 = __floats2bfloat162_rn(wj, wj);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(sWX + sw128(row, ch0 + q)) =
                        scale_bf16x8(*reinterpret_cast<const uint4*>(xs + sw128(row, ch0 + q)), w2);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                mbar_arrive(bar_sready);
                if (idx > 0) y_epilogue(idx - 1, true);
                else mbar_arrive(bar_yread);
                mbar_wait_bounded(bar_m1, ph, kWaitNs, aborted, prm.status);
                mbar_wait_bounded(bar_myo, ph, kWaitNs, aborted, prm.status);
                tc_fence_before_sync();
                mbar_arrive(bar_mready);   // (no masked tiles)
                if (it.pre_last) {
                    const bool from_start = rg.startC - rg.npre == 0;
                    pre_ok = from_start || both_cut;
                    mbar_wait_bounded(bar_m4, ph, kWaitNs, aborted, prm.status);
                    tc_fence_after_sync();
                    if (from_start && prm.init_state) {
                        // + the initial state decayed over the walk, 16 columns at a time
                        const int seq = (int)prm.fH.div((uint32_t)it.chain);
                        const float* src =
                            prm.init_state + ((size_t)seq * Hf + 2 * (it.chain - seq * prm.H) + hd) * kPN;
                        const float d0 = ex2_approx(lsum);
#pragma unroll 1
                        for (int hp = 0; hp < 32; hp += 16) {
                            float hs[16];
                            tmem_ld16(tH + (uint32_t)hp, hs);
                            tmem_wait_ld();
#pragma unroll
                            for (int p = 0; p < 16; ++p) hs[p] = fmaf(d0, src[(size_t)(pq + hp + p) * kN + row], hs[p]);
                            tmem_st16(tH + (uint32_t)hp, hs);
                            tmem_wait_st();
                        }
                    }
                }
                prev_pre = true;
                continue;
            }

            // 1. the state entering item idx (fp32; this thread's head, 32
            //    columns p of state column n = row)
            float hv[32];
            if (it.seg_start) {
                segment_state(it, hv);
            } else {
                // the previous state product is done (w o X is free), and
                // so is its C h^T (waited for before its masked tiles were
                // released), so the bf16 state may be rewritten
                mbar_wait_bounded(bar_m4, (uint32_t)(idx - 1) & 1u, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                pair_ld32(tH, hv);
                tmem_wait_ld();
            }
            // 2. its bf16 copy for C h^T
#pragma unroll
            for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(sHB + sw128(row, ch0 + q)) = pack_bf16x8(&hv[q * 8]);
            // 3. the decayed state back into TMEM and w o X
            mbar_wait_bounded(bar_vec, ph, kWaitNs, aborted, prm.status);
            const float cl_i = cv[row];
            const float cl_last = cv[kQ - 1];
            {
                const float decay = ex2_approx(cl_last);
#pragma unroll
                for (int p = 0; p < 32; p += 2) {
                    const float2 r = mul2(make_float2(hv[p], hv[p + 1]), make_float2(decay, decay));
                    hv[p] = r.x;
                    hv[p + 1] = r.y;
                }
                pair_st32(tH, hv);
            }
            mbar_wait_bounded(bar_ldx + (idx & 1), (uint32_t)(idx >> 1) & 1u, kWaitNs, aborted, prm.status);
            {
                const float wj = ex2_approx(cl_last - cl_i) * cv[kQ + row];
                const __nv_bfloat162 w2 = __floats2bfloat162_rn(wj, wj);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(sWX + sw128(row, ch0 + q)) =
                        scale_bf16x8(*reinterpret_cast<const uint4*>(xs + sw128(row, ch0 + q)), w2);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(bar_sready);   // the state product can start

            // 4. y of the previous item; then C h^T of this one may go into Y
            if (idx > 0) y_epilogue(idx - 1, true);
            else mbar_arrive(bar_yread);

            // 5. both heads' masked tiles from one read of G (column block jb
            //    is zero above the row quadrant's diagonal block; of every
            //    block, column quarter `quarter` takes 8 columns).  The
            //    blocks go one at a time through a loop that is not unrolled:
            //    the smaller code (one copy of each block form) is faster
            //    than loading all four blocks at once (8B layer 0.229 ->
            //    0.215 ms).
            mbar_wait_bounded(bar_m1, ph, kWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            {
                const float* cm0 = vecs(idx & 1, 0);
                const float* cm1 = vecs(idx & 1, 1);
                const float cl0 = cm0[row], cl1 = cm1[row];
                const float Dm0 = prm.D ? prm.D[h0] : 0.0f, Dm1 = prm.D ? prm.D[h0 + 1] : 0.0f;
#pragma unroll 1
                for (int jb = 0; jb < 4; ++jb) {
                    const int j0 = jb * 32 + quarter * 8;
                    uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u};
                    if (jb <= quad) {
                        float gv[8];
                        tmem_ld8(tmem + pr::kColG + lane_off + (uint32_t)j0, gv);
                        tmem_wait_ld();
#pragma unroll
                        for (int hm = 0; hm < 2; ++hm) {
                            const float* cm = hm ? cm1 : cm0;
                            const float cl_m = hm ? cl1 : cl0;
                            const float Dm = hm ? Dm1 : Dm0;
                            uint32_t* w = hm ? w1 : w0;
                            if (jb < quad) {
                                const float u = ex2_approx(cl_m - cm[jb * 32 + 31]);
                                const float4 va = reinterpret_cast<const float4*>(cm + 2 * kQ + j0)[0];
                                const float4 vb = reinterpret_cast<const float4*>(cm + 2 * kQ + j0)[1];
                                const float vv8[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 uv = mul2(make_float2(u, u), make_float2(vv8[2 * e], vv8[2 * e + 1]));
                                    const float2 m = mul2(make_float2(gv[2 * e], gv[2 * e + 1]), uv);
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(m.x, m.y);
                                    w[e] = *reinterpret_cast<uint32_t*>(&b2);
                                }
                            } else {
                                const float4 ca = reinterpret_cast<const float4*>(cm + j0)[0];
                                const float4 cb = reinterpret_cast<const float4*>(cm + j0)[1];
                                const float4 da = reinterpret_cast<const float4*>(cm + kQ + j0)[0];
                                const float4 db = reinterpret_cast<const float4*>(cm + kQ + j0)[1];
                                const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                                const float dd[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
                                float m[8];
#pragma unroll
                                for (int e = 0; e < 8; e += 2) {
                                    const float2 f = mul2(make_float2(ex2_approx(cl_m - cc[e]), ex2_approx(cl_m - cc[e + 1])),
                                                          make_float2(dd[e], dd[e + 1]));
                                    const float2 v = mul2(make_float2(gv[e], gv[e + 1]), f);
                                    m[e] = (j0 + e < row) ? v.x : (j0 + e == row ? v.x + Dm : 0.0f);
                                    m[e + 1] = (j0 + e + 1 < row) ? v.y : (j0 + e + 1 == row ? v.y + Dm : 0.0f);
                                }
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(m[2 * e], m[2 * e + 1]);
                                    w[e] = *reinterpret_cast<uint32_t*>(&b2);
                                }
                            }
                        }
                    }
                    tmem_st4(tmem + pr::kColM + lane_off + (uint32_t)(j0 >> 1), w0[0], w0[1], w0[2], w0[3]);
                    tmem_st4(tmem + pr::kColM + 64u + lane_off + (uint32_t)(j0 >> 1), w1[0], w1[1], w1[2], w1[3]);
                }
            }
            // 6. C h^T of this thread's head and columns scaled by 2^(cl_i)
            //    in place: M X accumulates onto it
            mbar_wait_bounded(bar_myo, ph, kWaitNs, aborted, prm.status);
            tc_fence_after_sync();
            {
                float yo[32];
                pair_ld32(tY, yo);
                tmem_wait_ld();
                const float sc = ex2_approx(cl_i);
#pragma unroll
                for (int p = 0; p < 32; p += 2) {
                    const float2 r = mul2(make_float2(yo[p], yo[p + 1]), make_float2(sc, sc));
                    yo[p] = r.x;
                    yo[p + 1] = r.y;
                }
                pair_st32(tY, yo);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_mready);   // M X can start

            // 7. end of a segment: the states leave the chip
            if (it.seg_end) {
                mbar_wait_bounded(bar_m4, ph, kWaitNs, aborted, prm.status);
                tc_fence_after_sync();
                pair_ld32(tH, hv);
                tmem_wait_ld();
                if (it.publish) {
                    float* dst = prm.ws_states + ((size_t)ticket * 2 + hd) * kPN;
#pragma unroll
                    for (int p = 0; p < 32; ++p) __stcg(dst + (size_t)(pq + p) * kN + row, hv[p]);
                    __threadfence();
                    named_bar_sync(kEwBarrier, kEwThreads);
                    if (tid == 0) st_release_gpu(prm.ws_ctrl + 16 + ticket, 1);
                } else if (prm.final_state) {
                    float* dst = prm.final_state + ((size_t)it.seq * Hf + h0 + hd) * kPN;
#pragma unroll
                    for (int p = 0; p < 32; ++p) dst[(size_t)(pq + p) * kN + row] = hv[p];
                }
            }
            prev_pre = false;
        }
        if (rg.count > 0) y_epilogue(rg.count - 1, false);
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
                     uint64_t row_bytes, uint32_t box_rows = kQ)
{
    auto fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {channels, L, b};
    const cuuint64_t strides[2] = {row_bytes, row_bytes * L};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}


// CTAs of the persistent grid (one per SM at most).  With at least as many
// chains as SMs every SM gets work from whole chains and their cuts.  With
// fewer chains, long ones are split further and the ranges that start
// inside a chain rebuild their starting state (*long_chains): a dense batch
// cuts every chain into the same number s of equal ranges (s chains' worth
// of SMs each, ranges of at least kMinRangeLong units), so that the heads of
// a group walk the same chunks at the same time and their shared B and C
// tiles come from HBM once and from L2 for the others (on the 1 x 32768-token,
// 64-head workload: 128 CTAs, 12% faster than 148 unaligned ones).  A ragged
// batch's chain lengths are known on the device only: it takes ranges of at
// least kMinRangeLong units over H times the chunks of its packed tokens.
// Dense batches whose groups hold an even number of heads run the head-pair
// kernel, whose chains are (sequence, head pair).
bool tc_pairs(const ScanArgs& a) { return !a.cu_seqlens && a.G > 0 && (a.H / a.G) % 2 == 0; }

int tc_slots(const ScanArgs& a, bool* long_chains = nullptr)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    const long long chains = (long long)(a.cu_seqlens ? a.nseq : a.b) * (tc_pairs(a) ? a.H / 2 : a.H);
    const long long nc = (a.L + kQ - 1) / kQ;
    const long long units = a.cu_seqlens ? (long long)a.H * nc : chains * nc;
    long long slots = chains < sms ? chains : sms;
    bool split_chains = false;
    if (a.cu_seqlens) {
        const long long split = units / kMinRangeLong;
        split_chains = chains < sms && split > chains;
        if (split_chains) slots = split < sms ? split : sms;
    } else if (chains < sms) {
        long long s_per = sms / chains;
        if (s_per > nc / kMinRangeLong) s_per = nc / kMinRangeLong;
        split_chains = s_per >= 2;
        if (split_chains) slots = chains * s_per;
    }
    if (long_chains) *long_chains = split_chains;
    return (int)slots;
}

}  // namespace

bool chunk_scan_tc_supported(const ScanArgs& a)
{
    return a.bf16 && a.P == kP && a.N == kN && a.Q == kQ;
}

size_t chunk_scan_tc_workspace_bytes(const ScanArgs& a)
{
    if (a.cu_seqlens) {   // ragged: the unit table comes first
        if (a.nseq <= 0) return 0;
        const int slots = tc_slots(a);
        return varlen_table_bytes(a.nseq) + varlen_desc_bytes(a.nseq, a.L, a.H, kQ) + kWsCtrlBytes(slots) +
               (size_t)slots * kStateBytes;
    }
    if (a.b <= 0 || a.L <= 0) return 0;
    const int slots = tc_slots(a);
    return kWsCtrlBytes(slots) + (size_t)slots * kStateBytes * (tc_pairs(a) ? 2 : 1);
}

cudaError_t launch_chunk_scan_tc(const ScanArgs& a, cudaStream_t s)
{
    CUtensorMap tmX, tmB, tmC;
    const uint64_t rb = (uint64_t)a.row_stride * 2;
    cudaError_t e;
    if ((e = make_map(&tmX, a.x, (uint64_t)a.H * a.P, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = make_map(&tmB, a.B, (uint64_t)a.G * a.N, a.L, a.b, rb)) != cudaSuccess) return e;
    if ((e = make_map(&tmC, a.C, (uint64_t)a.G * a.N, a.L, a.b, rb)) != cudaSuccess) return e;
    CUtensorMap tmY;
    if ((e = make_map(&tmY, a.y, (uint64_t)a.H * a.P, a.L, a.b, (uint64_t)a.H * a.P * 2)) != cudaSuccess) return e;
    YBoxes ypart{};   // (used by ragged batches only)
    if (a.cu_seqlens) {   // a ragged batch's partial last chunks
        for (int q = 0; q < 4; ++q)
            if ((e = make_map(&ypart.m[q], a.y, (uint64_t)a.H * a.P, a.L, a.b, (uint64_t)a.H * a.P * 2,
                              (uint32_t)(64 >> q))) != cudaSuccess)
                return e;
    }
    bool long_chains = false;
    const int slots = tc_slots(a, &long_chains);
    const bool pairs = tc_pairs(a);
    const int hunits = pairs ? a.H / 2 : a.H;   // chains per sequence
    auto kernel = pairs ? (long_chains ? chunk_scan_tc_pair_kernel<true> : chunk_scan_tc_pair_kernel<false>)
                  : a.cu_seqlens
                      ? (long_chains ? chunk_scan_tc_kernel<true, true> : chunk_scan_tc_kernel<true, false>)
                      : (long_chains ? chunk_scan_tc_kernel<false, true> : chunk_scan_tc_kernel<false, false>);
    const int smem_bytes = pairs ? pr::kSmemBytes : kSmemBytes;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    const size_t ctrl = kWsCtrlBytes(slots);
    const bool ragged = a.cu_seqlens != nullptr;
    // a ragged batch: header and sequence table, then the unit descriptors
    const size_t vtab = ragged ? varlen_table_bytes(a.nseq) : 0;
    const size_t table = ragged ? vtab + varlen_desc_bytes(a.nseq, a.L, a.H, kQ) : 0;
    if (!a.workspace || a.workspace_bytes < table + ctrl + (size_t)slots * kStateBytes * (pairs ? 2 : 1))
        return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    int* ws_ctrl = reinterpret_cast<int*>(ws + table);
    // ticket counter and hand-off flags start at zero on every call (a
    // ragged call's preparation kernel clears them with its other work)
    if (ragged) {
        e = launch_varlen_prep(a.cu_seqlens, a.nseq, a.L, a.H, kQ, reinterpret_cast<int*>(ws),
                               reinterpret_cast<int*>(ws + kVarlenUnitsOffset), ws_ctrl, (int)(ctrl / 4),
                               a.init_state, a.final_state, (long long)a.H * kP * kN, a.status, s);
        if (e != cudaSuccess) return e;
    } else if ((e = cudaMemsetAsync(ws_ctrl, 0, ctrl, s)) != cudaSuccess) {
        return e;
    }
    Params prm;
    prm.dt_raw = static_cast<const __nv_bfloat16*>(a.dt_raw);
    prm.dt_bias = a.dt_bias;
    prm.A = a.A;
    prm.D = a.D;
    prm.init_state = a.init_state;
    prm.y = static_cast<__nv_bfloat16*>(a.y);
    prm.final_state = a.final_state;
    prm.L = a.L;
    prm.H = hunits;
    prm.Hf = a.H;
    prm.G = a.G;
    prm.nc = ragged ? 1 : (a.L + kQ - 1) / kQ;   // (a ragged batch's chunk counts vary)
    prm.nslots = slots;
    prm.units = ragged ? 0 : a.b * hunits * prm.nc;
    prm.fnc = FastDiv::make((uint32_t)prm.nc);
    prm.fH = FastDiv::make((uint32_t)hunits);
    prm.fHG = FastDiv::make((uint32_t)(hunits / a.G));
    prm.ws_ctrl = ws_ctrl;
    prm.ws_states = reinterpret_cast<float*>(ws + table + ctrl);
    prm.cu_seqlens = a.cu_seqlens;
    prm.seq_units = ragged ? reinterpret_cast<const int*>(ws + kVarlenUnitsOffset) : nullptr;
    prm.ws_hdr = ragged ? reinterpret_cast<const int*>(ws) : nullptr;
    prm.unit_desc = ragged ? reinterpret_cast<int4*>(ws + vtab) : nullptr;
    prm.nseq = ragged ? a.nseq : a.b;
    prm.status = a.status;
    kernel<<<slots, kThreads, smem_bytes, s>>>(tmX, tmB, tmC, tmY, ypart, prm);
    return cudaGetLastError();
}

}  // namespace ssd
