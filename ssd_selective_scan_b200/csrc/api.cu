// api.cu -- the extern "C" entry points of libssd (declared in include/ssd.h):
// argument validation, kernel selection and launch.  No allocation, no
// synchronisation, no global mutable state.
#include "ssd.h"

#include <cuda_bf16.h>

#include "kernels.h"
#include "decode.h"
#include "scan_bwd.h"

namespace {

using ssd::ScanArgs;

struct Range {
    uintptr_t lo, hi;   // [lo, hi)
};

Range span(const void* p, int64_t bytes)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + (uintptr_t)(bytes > 0 ? bytes : 0)};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

bool valid_dtype(ssd_dtype_t d) { return d == SSD_F32 || d == SSD_BF16; }

int elem_bytes(ssd_dtype_t d) { return d == SSD_F32 ? 4 : 2; }

ssd_status_t from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return SSD_OK;
    (void)cudaGetLastError();
    return SSD_ERR_CUDA;
}

int max_optin_smem()
{
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
    return v;
}

size_t round_up_256(size_t n) { return (n + 255) / 256 * 256; }

}  // namespace

extern "C" {

const char* ssd_status_string(ssd_status_t s)
{
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument (nothing launched)";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: no kernel for this combination (nothing launched)";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: kernel launch failed";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "SSD_ERR_UNKNOWN";
}

int ssd_abi_version(void) { return SSD_ABI_VERSION; }

ssd_status_t ssd_conv1d_silu(const void* xBC, void* out, const float* w, const float* bias,
                             void* conv_state, int b, int L, int conv_dim, int k,
                             ssd_dtype_t dtype, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || L < 0 || conv_dim <= 0 || k <= 0) return SSD_ERR_INVALID_ARG;
    if (b == 0 || L == 0) return SSD_OK;   // empty work: nothing is read or written
    if (!xBC || !out || !w) return SSD_ERR_INVALID_ARG;
    const int e = elem_bytes(dtype);
    const int vec = 16 / e;
    if (conv_dim % vec) return SSD_ERR_INVALID_ARG;
    if (!aligned(xBC, 16) || !aligned(out, 16) || !aligned(w, 16) || (bias && !aligned(bias, 4)) ||
        (conv_state && !aligned(conv_state, 16)))
        return SSD_ERR_INVALID_ARG;
    const int64_t io_bytes = (int64_t)b * L * conv_dim * e;
    const Range rx = span(xBC, io_bytes), ro = span(out, io_bytes);
    const Range rs = span(conv_state, conv_state ? (int64_t)b * conv_dim * k * e : 0);
    if (overlap(rx, ro) || overlap(rs, rx) || overlap(rs, ro)) return SSD_ERR_INVALID_ARG;
    if (k < 2 || k > 4) return SSD_ERR_UNSUPPORTED;
    if (b > 65535 || (L + 31) / 32 > 65535) return SSD_ERR_UNSUPPORTED;
    return from_cuda(ssd::launch_conv1d_silu(xBC, out, w, bias, conv_state, b, L, conv_dim, k,
                                             dtype == SSD_BF16, stream));
}

size_t ssd_chunk_scan_workspace_bytes(int b, int L, int H, int P, int N, int G, int Q,
                                      ssd_dtype_t dtype)
{
    if (b <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || !valid_dtype(dtype)) return 0;
    ScanArgs a{};
    a.b = b; a.L = L; a.H = H; a.P = P; a.N = N; a.G = G; a.Q = Q;
    a.bf16 = dtype == SSD_BF16;
    return ssd::chunk_scan_tc_supported(a) ? ssd::chunk_scan_tc_workspace_bytes(a) : 0;
}

ssd_status_t ssd_chunk_scan_fwd(const void* x, const void* B, const void* C, int64_t row_stride,
                                const void* dt_raw, const float* dt_bias, const float* A,
                                const float* D, const float* init_state, void* y,
                                float* final_state, int b, int L, int H, int P, int N, int G,
                                int Q, ssd_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                int32_t* status, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0)
        return SSD_ERR_INVALID_ARG;
    if (H % G || P % 8 || N % 8 || (Q != 64 && Q != 128)) return SSD_ERR_INVALID_ARG;
    // With no tokens the token tensors are never touched and may be NULL.
    const bool tokens = b > 0 && L > 0;
    if (!A || (tokens && (!x || !B || !C || !dt_raw || !y))) return SSD_ERR_INVALID_ARG;
    if (row_stride % 8 || row_stride < (int64_t)H * P || row_stride < (int64_t)G * N)
        return SSD_ERR_INVALID_ARG;
    const void* ptrs16[] = {x, B, C, dt_raw, y, init_state, final_state};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return SSD_ERR_INVALID_ARG;
    if (!aligned(A, 4) || (dt_bias && !aligned(dt_bias, 4)) || (D && !aligned(D, 4)) ||
        (status && !aligned(status, 4)))
        return SSD_ERR_INVALID_ARG;
    const size_t need_ws = ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype);
    if (workspace_bytes < need_ws || (need_ws && !workspace)) return SSD_ERR_INVALID_ARG;

    const int e = elem_bytes(dtype);
    const int64_t rows = (int64_t)b * L;
    const int64_t row_bytes = row_stride * e;
    // Conservative extents of the strided inputs: from the pointer to the end
    // of the last row's channel range.
    const Range rx = span(x, rows ? (rows - 1) * row_bytes + (int64_t)H * P * e : 0);
    const Range rB = span(B, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rC = span(C, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rdt = span(dt_raw, rows * H * e);
    const Range ry = span(y, rows * H * P * e);
    const int64_t st_bytes = (int64_t)b * H * P * N * 4;
    const Range ri = span(init_state, init_state ? st_bytes : 0);
    const Range rf = span(final_state, final_state ? st_bytes : 0);
    const Range rw = span(workspace, (int64_t)workspace_bytes);
    for (Range in : {rx, rB, rC, rdt, ri})
        if (overlap(ry, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rB, rC, rdt, ry})
        if (overlap(rf, in)) return SSD_ERR_INVALID_ARG;
    if (final_state && init_state && final_state != init_state && overlap(rf, ri))
        return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rB, rC, rdt, ry, ri, rf})
        if (overlap(rw, in)) return SSD_ERR_INVALID_ARG;

    if (b == 0) return SSD_OK;
    if (L == 0) {
        // No tokens: the final state is the initial state.
        if (!final_state || final_state == init_state) return SSD_OK;
        return from_cuda(init_state ? cudaMemcpyAsync(final_state, init_state, (size_t)st_bytes,
                                                      cudaMemcpyDeviceToDevice, stream)
                                    : cudaMemsetAsync(final_state, 0, (size_t)st_bytes, stream));
    }
    // the unit list of the tensor-core path: b * H * chunks
    if ((int64_t)b * H * ((L + Q - 1) / Q) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;

    ScanArgs a{x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y, final_state,
               b, L, H, P, N, G, Q, dtype == SSD_BF16, workspace, workspace_bytes, status};
    if (ssd::chunk_scan_tc_supported(a)) return from_cuda(ssd::launch_chunk_scan_tc(a, stream));
    if (ssd::chunk_scan_simt_smem_bytes(P, N) > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
    return from_cuda(ssd::launch_chunk_scan_simt(a, stream));
}

size_t ssd_chunk_scan_varlen_workspace_bytes(int nseq, int T, int H, int P, int N, int G, int Q,
                                             ssd_dtype_t dtype)
{
    if (nseq <= 0 || T < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || !valid_dtype(dtype)) return 0;
    static const int kAnyPtr = 0;
    ScanArgs a{};
    a.b = 1; a.L = T; a.H = H; a.P = P; a.N = N; a.G = G; a.Q = Q;
    a.bf16 = dtype == SSD_BF16;
    a.cu_seqlens = &kAnyPtr;   // only its presence matters here
    a.nseq = nseq;
    return ssd::chunk_scan_tc_supported(a) ? ssd::chunk_scan_tc_workspace_bytes(a) : ssd::varlen_table_bytes(nseq);
}

ssd_status_t ssd_chunk_scan_fwd_varlen(const void* x, const void* B, const void* C, int64_t row_stride,
                                       const void* dt_raw, const float* dt_bias, const float* A,
                                       const float* D, const float* init_state, void* y,
                                       float* final_state, const int32_t* cu_seqlens, int nseq, int T,
                                       int H, int P, int N, int G, int Q, ssd_dtype_t dtype, void* workspace,
                                       size_t workspace_bytes, int32_t* status, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || nseq < 0 || T < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0)
        return SSD_ERR_INVALID_ARG;
    if (H % G || P % 8 || N % 8 || (Q != 64 && Q != 128)) return SSD_ERR_INVALID_ARG;
    if (nseq == 0) return T == 0 ? SSD_OK : SSD_ERR_INVALID_ARG;   // tokens without sequences
    // cu_seqlens is read on the device; a bad one is reported through status
    if (!A || !cu_seqlens || !status) return SSD_ERR_INVALID_ARG;
    const bool tokens = T > 0;
    if (tokens && (!x || !B || !C || !dt_raw || !y)) return SSD_ERR_INVALID_ARG;
    if (row_stride % 8 || row_stride < (int64_t)H * P || row_stride < (int64_t)G * N) return SSD_ERR_INVALID_ARG;
    const void* ptrs16[] = {x, B, C, dt_raw, y, init_state, final_state};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return SSD_ERR_INVALID_ARG;
    if (!aligned(A, 4) || (dt_bias && !aligned(dt_bias, 4)) || (D && !aligned(D, 4)) || !aligned(status, 4) ||
        !aligned(cu_seqlens, 4))
        return SSD_ERR_INVALID_ARG;
    // the unit list of the tensor-core path: H * (T / Q + nseq) bounds it
    if ((int64_t)H * ((int64_t)T / Q + nseq + 1) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    const size_t need_ws = ssd_chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, dtype);
    if (workspace_bytes < need_ws || !workspace) return SSD_ERR_INVALID_ARG;

    const int e = elem_bytes(dtype);
    const int64_t rows = T;
    const int64_t row_bytes = row_stride * e;
    const Range rx = span(x, rows ? (rows - 1) * row_bytes + (int64_t)H * P * e : 0);
    const Range rB = span(B, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rC = span(C, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rdt = span(dt_raw, rows * H * e);
    const Range ry = span(y, rows * H * P * e);
    const int64_t st_bytes = (int64_t)nseq * H * P * N * 4;
    const Range ri = span(init_state, init_state ? st_bytes : 0);
    const Range rf = span(final_state, final_state ? st_bytes : 0);
    const Range rcu = span(cu_seqlens, (int64_t)(nseq + 1) * 4);
    const Range rw = span(workspace, (int64_t)workspace_bytes);
    for (Range in : {rx, rB, rC, rdt, ri, rcu})
        if (overlap(ry, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rB, rC, rdt, ry, rcu})
        if (overlap(rf, in)) return SSD_ERR_INVALID_ARG;
    if (final_state && init_state && final_state != init_state && overlap(rf, ri)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rB, rC, rdt, ry, ri, rf, rcu})
        if (overlap(rw, in)) return SSD_ERR_INVALID_ARG;

    if (!tokens) {
        // every sequence is empty: check cu_seqlens and set the final states
        return from_cuda(ssd::launch_varlen_prep(reinterpret_cast<const int*>(cu_seqlens), nseq, 0, H, Q,
                                                 static_cast<int*>(workspace), nullptr, nullptr, 0, init_state,
                                                 final_state, (long long)H * P * N, status, stream));
    }
    ScanArgs a{x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y, final_state,
               1, T, H, P, N, G, Q, dtype == SSD_BF16, workspace, workspace_bytes, status};
    a.cu_seqlens = reinterpret_cast<const int*>(cu_seqlens);
    a.nseq = nseq;
    if (ssd::chunk_scan_tc_supported(a)) return from_cuda(ssd::launch_chunk_scan_tc(a, stream));
    if (ssd::chunk_scan_simt_smem_bytes(P, N) > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
    return from_cuda(ssd::launch_chunk_scan_simt(a, stream));
}

size_t ssd_conv_scan_workspace_bytes(int b, int L, int H, int P, int N, int G, int Q, int k,
                                     ssd_dtype_t dtype)
{
    if (b <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || k <= 0 || !valid_dtype(dtype)) return 0;
    const size_t conv_dim = (size_t)H * P + 2 * (size_t)G * N;
    return round_up_256((size_t)b * L * conv_dim * elem_bytes(dtype)) +
           ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype);
}

ssd_status_t ssd_conv_scan_fwd(const void* xBC, const float* w, const float* bias, void* conv_state,
                               const void* dt_raw, const float* dt_bias, const float* A, const float* D,
                               const float* init_state, void* y, float* final_state, int b, int L, int H,
                               int P, int N, int G, int Q, int k, ssd_dtype_t dtype, void* workspace,
                               size_t workspace_bytes, int32_t* status, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || k <= 0)
        return SSD_ERR_INVALID_ARG;
    if (H % G || P % 8 || N % 8 || (Q != 64 && Q != 128)) return SSD_ERR_INVALID_ARG;
    if ((int64_t)H * P + 2 * (int64_t)G * N > 0x7fffffffLL) return SSD_ERR_INVALID_ARG;
    const int conv_dim = H * P + 2 * G * N;   // a multiple of 8: 16-byte rows for either dtype
    if (b == 0 || L == 0) {
        // no tokens: the conv cache is unchanged and the scan's rule for
        // empty sequences applies (final state = initial state)
        if (k > 4 || k < 2) return SSD_ERR_UNSUPPORTED;
        return ssd_chunk_scan_fwd(nullptr, nullptr, nullptr, conv_dim, nullptr, dt_bias, A, D, init_state, nullptr,
                                  final_state, b, L, H, P, N, G, Q, dtype, nullptr, 0, status, stream);
    }
    if (!xBC || !w || !dt_raw || !A || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs16[] = {xBC, w, conv_state, dt_raw, y, init_state, final_state, workspace};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return SSD_ERR_INVALID_ARG;
    if (!aligned(A, 4) || (bias && !aligned(bias, 4)) || (dt_bias && !aligned(dt_bias, 4)) || (D && !aligned(D, 4)) ||
        (status && !aligned(status, 4)))
        return SSD_ERR_INVALID_ARG;
    const size_t need_ws = ssd_conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, dtype);
    if (workspace_bytes < need_ws || !workspace) return SSD_ERR_INVALID_ARG;

    const int e = elem_bytes(dtype);
    const int64_t rows = (int64_t)b * L;
    const Range rx = span(xBC, rows * conv_dim * e);
    const Range rw = span(w, (int64_t)conv_dim * k * 4);
    const Range rcs = span(conv_state, conv_state ? (int64_t)b * conv_dim * k * e : 0);
    const Range rdt = span(dt_raw, rows * H * e);
    const Range ry = span(y, rows * H * P * e);
    const int64_t st_bytes = (int64_t)b * H * P * N * 4;
    const Range ri = span(init_state, init_state ? st_bytes : 0);
    const Range rf = span(final_state, final_state ? st_bytes : 0);
    const Range rws = span(workspace, (int64_t)workspace_bytes);
    for (Range in : {rx, rw, rcs, rdt, ri})
        if (overlap(ry, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rw, rcs, rdt, ry})
        if (overlap(rf, in)) return SSD_ERR_INVALID_ARG;
    if (final_state && init_state && final_state != init_state && overlap(rf, ri)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rw, rdt, ry, ri, rf})
        if (overlap(rcs, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rw, rcs, rdt, ry, ri, rf})
        if (overlap(rws, in)) return SSD_ERR_INVALID_ARG;
    if (k < 2 || k > 4) return SSD_ERR_UNSUPPORTED;
    if (b > 65535 || (L + 31) / 32 > 65535) return SSD_ERR_UNSUPPORTED;
    if ((int64_t)b * H * ((L + Q - 1) / Q) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;

    // the conv output u into the workspace, then the scan on its x | B | C
    // channel ranges (row stride conv_dim)
    const bool bf16 = dtype == SSD_BF16;
    const int GN = G * N, HP = H * P;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    ScanArgs a{nullptr, nullptr, nullptr, conv_dim, dt_raw, dt_bias, A, D, init_state, y, final_state,
               b, L, H, P, N, G, Q, bf16, nullptr, 0, status};
    const bool tc = ssd::chunk_scan_tc_supported(a);
    if (!tc && ssd::chunk_scan_simt_smem_bytes(P, N) > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
    const size_t u_bytes = round_up_256((size_t)rows * conv_dim * e);
    const ssd_status_t st = from_cuda(ssd::launch_conv1d_silu(xBC, ws, w, bias, conv_state, b, L, conv_dim, k, bf16, stream));
    if (st != SSD_OK) return st;
    a.x = ws;
    a.B = ws + (size_t)HP * e;
    a.C = ws + (size_t)(HP + GN) * e;
    a.workspace = ws + u_bytes;
    a.workspace_bytes = workspace_bytes - u_bytes;
    return from_cuda(tc ? ssd::launch_chunk_scan_tc(a, stream) : ssd::launch_chunk_scan_simt(a, stream));
}

ssd_status_t ssd_state_update(float* state, const void* x, const void* B, const void* C,
                              int64_t row_stride, const void* dt_raw, const float* dt_bias,
                              const float* A, const float* D, void* y, int b, int H, int P, int N,
                              int G, ssd_dtype_t dtype, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G)
        return SSD_ERR_INVALID_ARG;
    if (!state || !x || !B || !C || !dt_raw || !A || !y) return SSD_ERR_INVALID_ARG;
    if (N % 4 || row_stride < (int64_t)H * P || row_stride < (int64_t)G * N) return SSD_ERR_INVALID_ARG;
    const int e = elem_bytes(dtype);
    if (!aligned(state, 16) || !aligned(x, e) || !aligned(B, e) || !aligned(C, e) ||
        !aligned(dt_raw, e) || !aligned(y, e) || !aligned(A, 4) || (dt_bias && !aligned(dt_bias, 4)) ||
        (D && !aligned(D, 4)))
        return SSD_ERR_INVALID_ARG;
    const Range rs = span(state, (int64_t)b * H * P * N * 4);
    const Range ry = span(y, (int64_t)b * H * P * e);
    const int64_t last = b ? (int64_t)(b - 1) * row_stride * e : 0;
    const Range rx = span(x, b ? last + (int64_t)H * P * e : 0);
    const Range rB = span(B, b ? last + (int64_t)G * N * e : 0);
    const Range rC = span(C, b ? last + (int64_t)G * N * e : 0);
    const Range rdt = span(dt_raw, (int64_t)b * H * e);
    for (Range in : {rx, rB, rC, rdt, ry})
        if (overlap(rs, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rB, rC, rdt})
        if (overlap(ry, in)) return SSD_ERR_INVALID_ARG;
    if (!ssd::state_update_supports_n(N)) return SSD_ERR_UNSUPPORTED;
    if ((int64_t)b * H > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    if (b == 0) return SSD_OK;
    return from_cuda(ssd::launch_state_update(state, x, B, C, row_stride, dt_raw, dt_bias, A, D, y,
                                              b, H, P, N, G, dtype == SSD_BF16, stream));
}

// Arguments of the decode step (both forms): SSD_OK, or the error to return
// (with b == 0 reported as SSD_OK and *nothing set).
static ssd_status_t decode_step_check(float* state, void* conv_state, const void* xBC, const float* w,
                                      const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                      const float* D, void* y, int b, int H, int P, int N, int G, int k,
                                      ssd_dtype_t dtype, const void* workspace, size_t workspace_bytes,
                                      bool with_workspace, bool* nothing)
{
    *nothing = false;
    if (!valid_dtype(dtype) || b < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || k <= 0 || H % G)
        return SSD_ERR_INVALID_ARG;
    if (N % 4) return SSD_ERR_INVALID_ARG;
    if ((int64_t)H * P + 2 * (int64_t)G * N > 0x7fffffffLL) return SSD_ERR_INVALID_ARG;
    if (b == 0) {
        *nothing = true;
        return SSD_OK;
    }
    if (!state || !conv_state || !xBC || !w || !dt_raw || !A || !y) return SSD_ERR_INVALID_ARG;
    const int e = elem_bytes(dtype);
    if (!aligned(state, 16) || !aligned(conv_state, e) || !aligned(xBC, e) || !aligned(dt_raw, e) ||
        !aligned(y, e) || !aligned(w, 4) || !aligned(A, 4) || (bias && !aligned(bias, 4)) ||
        (dt_bias && !aligned(dt_bias, 4)) || (D && !aligned(D, 4)))
        return SSD_ERR_INVALID_ARG;
    const int64_t conv_dim = (int64_t)H * P + 2 * (int64_t)G * N;
    const Range rs = span(state, (int64_t)b * H * P * N * 4);
    const Range rcs = span(conv_state, (int64_t)b * conv_dim * k * e);
    const Range rx = span(xBC, (int64_t)b * conv_dim * e);
    const Range rw = span(w, conv_dim * k * 4);
    const Range rdt = span(dt_raw, (int64_t)b * H * e);
    const Range ry = span(y, (int64_t)b * H * P * e);
    for (Range in : {rcs, rx, rw, rdt, ry})
        if (overlap(rs, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rw, rdt, ry})
        if (overlap(rcs, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rx, rw, rdt})
        if (overlap(ry, in)) return SSD_ERR_INVALID_ARG;
    if (with_workspace) {
        if (!workspace || !aligned(workspace, 4) || workspace_bytes < (size_t)b * G * 4) return SSD_ERR_INVALID_ARG;
        const Range rws = span(workspace, (int64_t)b * G * 4);
        for (Range in : {rs, rcs, rx, rw, rdt, ry})
            if (overlap(rws, in)) return SSD_ERR_INVALID_ARG;
    }
    if (k < 2 || k > 4 || !ssd::state_update_supports_n(N)) return SSD_ERR_UNSUPPORTED;
    if (with_workspace && P > ssd::decode_step_head_max_p()) return SSD_ERR_UNSUPPORTED;
    if ((int64_t)b * (with_workspace ? H : G) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    const size_t smem = with_workspace ? ssd::decode_step_head_smem_bytes(P, N) : ssd::decode_step_smem_bytes(H, P, N, G);
    if (smem > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

ssd_status_t ssd_decode_step(float* state, void* conv_state, const void* xBC, const float* w,
                             const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                             const float* D, void* y, int b, int H, int P, int N, int G, int k,
                             ssd_dtype_t dtype, cudaStream_t stream)
{
    bool nothing = false;
    const ssd_status_t st = decode_step_check(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N,
                                              G, k, dtype, nullptr, 0, false, &nothing);
    if (st != SSD_OK || nothing) return st;
    return from_cuda(ssd::launch_decode_step(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P,
                                             N, G, k, dtype == SSD_BF16, stream));
}

size_t ssd_decode_step_workspace_bytes(int b, int G)
{
    return b > 0 && G > 0 ? (size_t)b * G * 4 : 0;
}

ssd_status_t ssd_decode_step_ws(float* state, void* conv_state, const void* xBC, const float* w,
                                const float* bias, const void* dt_raw, const float* dt_bias, const float* A,
                                const float* D, void* y, int b, int H, int P, int N, int G, int k,
                                ssd_dtype_t dtype, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    bool nothing = false;
    const ssd_status_t st = decode_step_check(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N,
                                              G, k, dtype, workspace, workspace_bytes, true, &nothing);
    if (st != SSD_OK || nothing) return st;
    return from_cuda(ssd::launch_decode_step_head(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y,
                                                  static_cast<int*>(workspace), b, H, P, N, G, k, dtype == SSD_BF16,
                                                  stream));
}

ssd_status_t ssd_linear_bf16(const void* x, int64_t ldx, const void* w, int64_t ldw, void* y, int64_t ldy, int M,
                             int N, int K, int32_t* status, cudaStream_t stream)
{
    if (M < 0 || N <= 0 || K <= 0) return SSD_ERR_INVALID_ARG;
    if (M == 0) return SSD_OK;
    if (!x || !w || !y) return SSD_ERR_INVALID_ARG;
    if (ldx < K || ldw < K || ldy < N || ldx % 8 || ldw % 8 || ldy % 8 || N % 8 || K % 8) return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16) || (status && !aligned(status, 4)))
        return SSD_ERR_INVALID_ARG;
    const Range rx = span(x, ((int64_t)(M - 1) * ldx + K) * 2), rw = span(w, ((int64_t)(N - 1) * ldw + K) * 2);
    const Range ry = span(y, ((int64_t)(M - 1) * ldy + N) * 2);
    if (overlap(ry, rx) || overlap(ry, rw)) return SSD_ERR_INVALID_ARG;
    if (!ssd::gemm_bf16_tn_supported(M, N, K, ldx, ldw, 0)) return SSD_ERR_UNSUPPORTED;
    return from_cuda(ssd::launch_gemm_bf16_tn(x, ldx, w, ldw, y, ldy, nullptr, 0, M, N, K, 0, status, stream));
}

namespace {

// Workspace of the mixer: in_proj's z | xBC columns and its dt columns, the
// conv output (later reused for the normed y), the scan's y, then the scan's
// own workspace.  Byte offsets, each region 256-byte aligned.
struct MixerWs {
    size_t zxbc, dt, u, y, scan, total;
};

MixerWs mixer_ws(int b, int L, int H, int P, int N, int G, int Q)
{
    const size_t M = (size_t)b * L;
    const size_t d_inner = (size_t)H * P, conv_dim = d_inner + 2 * (size_t)G * N;
    MixerWs w{};
    w.zxbc = 0;
    w.dt = w.zxbc + round_up_256(M * (d_inner + conv_dim) * 2);
    w.u = w.dt + round_up_256(M * (size_t)H * 2);
    w.y = w.u + round_up_256(M * conv_dim * 2);
    w.scan = w.y + round_up_256(M * d_inner * 2);
    w.total = w.scan + ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, SSD_BF16);
    return w;
}

}  // namespace

size_t ssd_mixer_workspace_bytes(int b, int L, int d_model, int H, int P, int N, int G, int Q, int k,
                                 ssd_dtype_t dtype)
{
    if (b <= 0 || L <= 0 || d_model <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || k <= 0 || dtype != SSD_BF16)
        return 0;
    return mixer_ws(b, L, H, P, N, G, Q).total;
}

ssd_status_t ssd_mixer_fwd(const void* hidden, const void* W_in, const float* conv_w, const float* conv_bias,
                           void* conv_state, const float* dt_bias, const float* A, const float* D,
                           const float* norm_w, const void* W_out, const float* init_state, void* out,
                           float* final_state, int b, int L, int d_model, int H, int P, int N, int G, int Q, int k,
                           int norm_groups, float eps, ssd_dtype_t dtype, void* workspace, size_t workspace_bytes,
                           int32_t* status, cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || L < 0 || d_model <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || k <= 0 ||
        norm_groups <= 0 || !(eps >= 0.0f))
        return SSD_ERR_INVALID_ARG;
    if (H % G || P % 8 || N % 8 || (Q != 64 && Q != 128) || d_model % 8) return SSD_ERR_INVALID_ARG;
    const int64_t d_inner = (int64_t)H * P, conv_dim = d_inner + 2 * (int64_t)G * N;
    if (d_inner + conv_dim + H > 0x7fffffffLL || d_inner % norm_groups || (d_inner / norm_groups) % 8)
        return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_BF16 || H % 8) return SSD_ERR_UNSUPPORTED;   // bf16 projections; 16-byte dt rows
    if (k < 2 || k > 4) return SSD_ERR_UNSUPPORTED;
    if (b == 0 || L == 0) {
        // no tokens: the conv cache is unchanged and the final state is the initial one
        return ssd_chunk_scan_fwd(nullptr, nullptr, nullptr, conv_dim, nullptr, dt_bias, A, D, init_state, nullptr,
                                  final_state, b, L, H, P, N, G, Q, dtype, nullptr, 0, status, stream);
    }
    if (!hidden || !W_in || !conv_w || !A || !norm_w || !W_out || !out) return SSD_ERR_INVALID_ARG;
    const void* ptrs16[] = {hidden, W_in, conv_w, conv_state, norm_w, W_out, init_state, out, final_state, workspace};
    for (const void* p : ptrs16)
        if (p && !aligned(p, 16)) return SSD_ERR_INVALID_ARG;
    if ((conv_bias && !aligned(conv_bias, 4)) || (dt_bias && !aligned(dt_bias, 4)) || !aligned(A, 4) ||
        (D && !aligned(D, 4)) || (status && !aligned(status, 4)))
        return SSD_ERR_INVALID_ARG;
    const MixerWs ws = mixer_ws(b, L, H, P, N, G, Q);
    if (!workspace || workspace_bytes < ws.total) return SSD_ERR_INVALID_ARG;
    const int64_t M = (int64_t)b * L;
    const int64_t nproj = d_inner + conv_dim + H;
    const Range rh = span(hidden, M * d_model * 2), rwi = span(W_in, nproj * d_model * 2);
    const Range rwo = span(W_out, (int64_t)d_model * d_inner * 2), ro = span(out, M * d_model * 2);
    const Range rcs = span(conv_state, conv_state ? (int64_t)b * conv_dim * k * 2 : 0);
    const int64_t st_bytes = (int64_t)b * H * P * N * 4;
    const Range ri = span(init_state, init_state ? st_bytes : 0), rf = span(final_state, final_state ? st_bytes : 0);
    const Range rws = span(workspace, (int64_t)workspace_bytes);
    for (Range in : {rh, rwi, rwo, rcs, ri, rws})
        if (overlap(ro, in)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rh, rwi, rwo, rcs, ro, rws})
        if (overlap(rf, in)) return SSD_ERR_INVALID_ARG;
    if (final_state && init_state && final_state != init_state && overlap(rf, ri)) return SSD_ERR_INVALID_ARG;
    for (Range in : {rh, rwi, rwo, ri})
        if (overlap(rws, in) || overlap(rcs, in)) return SSD_ERR_INVALID_ARG;
    if (overlap(rws, rcs)) return SSD_ERR_INVALID_ARG;
    if (M > 0x7fffffffLL || b > 65535 || (L + 31) / 32 > 65535) return SSD_ERR_UNSUPPORTED;
    if ((int64_t)b * H * ((L + Q - 1) / Q) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    if (!ssd::gemm_bf16_tn_supported((int)M, (int)nproj, d_model, d_model, d_model, (int)(d_inner + conv_dim)) ||
        !ssd::gemm_bf16_tn_supported((int)M, d_model, (int)d_inner, d_inner, d_inner, 0))
        return SSD_ERR_UNSUPPORTED;

    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    auto* zxbc = reinterpret_cast<__nv_bfloat16*>(wsb + ws.zxbc);
    auto* dt = reinterpret_cast<__nv_bfloat16*>(wsb + ws.dt);
    auto* u = reinterpret_cast<__nv_bfloat16*>(wsb + ws.u);
    auto* ybuf = reinterpret_cast<__nv_bfloat16*>(wsb + ws.y);
    const int64_t ldz = d_inner + conv_dim;
    // 1. in_proj: z | xBC into one buffer, dt into another
    cudaError_t e = ssd::launch_gemm_bf16_tn(hidden, d_model, W_in, d_model, zxbc, ldz, dt, H, (int)M, (int)nproj,
                                             d_model, (int)ldz, status, stream);
    // 2. conv1d + SiLU of the xBC columns
    if (e == cudaSuccess)
        e = ssd::launch_conv1d_silu(zxbc + d_inner, u, conv_w, conv_bias, conv_state, b, L, (int)conv_dim, k, true,
                                    stream, ldz);
    // 3. the chunked scan
    if (e == cudaSuccess) {
        ScanArgs a{u, u + d_inner, u + d_inner + (int64_t)G * N, conv_dim, dt, dt_bias, A, D, init_state, ybuf,
                   final_state, b, L, H, P, N, G, Q, true, wsb + ws.scan, workspace_bytes - ws.scan, status};
        if (ssd::chunk_scan_tc_supported(a)) {
            e = ssd::launch_chunk_scan_tc(a, stream);
        } else {
            if (ssd::chunk_scan_simt_smem_bytes(P, N) > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
            e = ssd::launch_chunk_scan_simt(a, stream);
        }
    }
    // 4. the gated RMSNorm, into the (now free) conv-output buffer
    if (e == cudaSuccess)
        e = ssd::launch_rmsnorm_gated(ybuf, d_inner, zxbc, ldz, norm_w, u, d_inner, (int)M, (int)d_inner, norm_groups,
                                      eps, stream);
    // 5. out_proj
    if (e == cudaSuccess)
        e = ssd::launch_gemm_bf16_tn(u, d_inner, W_out, d_inner, out, d_model, nullptr, 0, (int)M, d_model,
                                     (int)d_inner, 0, status, stream);
    return from_cuda(e);
}

size_t ssd_chunk_scan_bwd_workspace_bytes(int b, int L, int H, int P, int N, int G, ssd_dtype_t dtype)
{
    if (b <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || !valid_dtype(dtype)) return 0;
    const size_t general = ssd::scan_bwd_workspace_bytes(b, L, H, P, N);
    // a tensor-core shape may still take the general path (unaligned pointers)
    if (ssd::scan_bwd_tc_shape(P, N, dtype == SSD_BF16))
        return std::max(general, ssd::scan_bwd_tc_workspace_bytes(b, L, H));
    return general;
}

ssd_status_t ssd_chunk_scan_bwd(const void* x, const void* B, const void* C, int64_t row_stride, const void* dt_raw,
                                const float* dt_bias, const float* A, const float* D, const float* init_state,
                                const void* dy, const float* dfinal, void* dx, void* dB, void* dC, void* ddt_raw,
                                float* dA, float* dD, float* ddt_bias, float* dinit, int b, int L, int H, int P,
                                int N, int G, ssd_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                cudaStream_t stream)
{
    if (!valid_dtype(dtype) || b < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G)
        return SSD_ERR_INVALID_ARG;
    if (!A || !dA || !dD || !ddt_bias) return SSD_ERR_INVALID_ARG;
    const bool tokens = b > 0 && L > 0;
    if (tokens && (!x || !B || !C || !dt_raw || !dy || !dx || !dB || !dC || !ddt_raw)) return SSD_ERR_INVALID_ARG;
    if (row_stride < (int64_t)H * P || row_stride < (int64_t)G * N) return SSD_ERR_INVALID_ARG;
    const int e = elem_bytes(dtype);
    const void* io_ptrs[] = {x, B, C, dt_raw, dy, dx, dB, dC, ddt_raw};
    for (const void* q : io_ptrs)
        if (q && !aligned(q, e)) return SSD_ERR_INVALID_ARG;
    const void* f32_ptrs[] = {dt_bias, A, D, init_state, dfinal, dA, dD, ddt_bias, dinit, workspace};
    for (const void* q : f32_ptrs)
        if (q && !aligned(q, 4)) return SSD_ERR_INVALID_ARG;
    const size_t need_ws = ssd_chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, dtype);
    if (workspace_bytes < need_ws || (need_ws && !workspace)) return SSD_ERR_INVALID_ARG;

    const int64_t rows = (int64_t)b * L;
    const int64_t row_bytes = row_stride * e;
    const Range rx = span(x, rows ? (rows - 1) * row_bytes + (int64_t)H * P * e : 0);
    const Range rB = span(B, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rC = span(C, rows ? (rows - 1) * row_bytes + (int64_t)G * N * e : 0);
    const Range rdt = span(dt_raw, rows * H * e);
    const Range rdy = span(dy, rows * H * P * e);
    const int64_t st_bytes = (int64_t)b * H * P * N * 4;
    const Range ri = span(init_state, init_state ? st_bytes : 0);
    const Range rfin = span(dfinal, dfinal ? st_bytes : 0);
    const Range rdx = span(dx, rows * H * P * e);
    const Range rdB = span(dB, rows * G * N * e);
    const Range rdC = span(dC, rows * G * N * e);
    const Range rddt = span(ddt_raw, rows * H * e);
    const Range rdA = span(dA, (int64_t)H * 4), rdD = span(dD, (int64_t)H * 4), rdb = span(ddt_bias, (int64_t)H * 4);
    const Range rdi = span(dinit, dinit ? st_bytes : 0);
    const Range rws = span(workspace, (int64_t)workspace_bytes);
    const Range ins[] = {rx, rB, rC, rdt, rdy, ri, rfin, span(A, (int64_t)H * 4)};
    const Range outs[] = {rdx, rdB, rdC, rddt, rdA, rdD, rdb, rdi, rws};
    for (int i = 0; i < 9; ++i) {
        for (const Range& in : ins)
            if (overlap(outs[i], in)) return SSD_ERR_INVALID_ARG;
        for (int j = i + 1; j < 9; ++j)
            if (overlap(outs[i], outs[j])) return SSD_ERR_INVALID_ARG;
    }
    if (!tokens) {
        // no tokens: the parameter gradients are zero and the initial
        // state's gradient is the final state's (or zero)
        cudaError_t err = cudaMemsetAsync(dA, 0, (size_t)H * 4, stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(dD, 0, (size_t)H * 4, stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(ddt_bias, 0, (size_t)H * 4, stream);
        if (err == cudaSuccess && dinit && b > 0)
            err = dfinal ? cudaMemcpyAsync(dinit, dfinal, (size_t)st_bytes, cudaMemcpyDeviceToDevice, stream)
                         : cudaMemsetAsync(dinit, 0, (size_t)st_bytes, stream);
        return from_cuda(err);
    }
    if ((int64_t)b * H > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    ssd::ScanBwdArgs a{x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, dy, dfinal, dx, dB, dC, ddt_raw,
                       dA, dD, ddt_bias, dinit, b, L, H, P, N, G, dtype == SSD_BF16, workspace};
    if (ssd::scan_bwd_tc_supported(a)) return from_cuda(ssd::launch_scan_bwd_tc(a, stream));
    if (ssd::scan_bwd_smem_bytes(P, N) > (size_t)max_optin_smem()) return SSD_ERR_UNSUPPORTED;
    return from_cuda(ssd::launch_scan_bwd(a, stream));
}

}  // extern "C"
