/*
 * ssd.h -- C ABI of libssd: the data-parallel hot path of the Mamba-2
 * selective state-space layer on NVIDIA B200 (sm_100a).
 *
 * Operations (sources are the pages this library implements):
 *   - causal depthwise conv1d + SiLU over the x | B | C channels, with a
 *     k-column rolling cache ("Hybrid Architectures for Language Models:
 *     Systematic Analysis and Design Insights", summary page, appendix C:
 *     the Mamba cache holds N_conv * (2*d_state + d_ssm) conv entries and
 *     d_ssm * d_state state entries per layer; Nemotron feasibility report,
 *     section 1.4: conv kernel 4, SiLU);
 *   - the chunked state-space-duality (SSD) scan: the recurrence
 *     h_t = Abar h_{t-1} + Bbar x_t, y_t = C h_t + D x_t (summary page,
 *     section 2 Background) evaluated chunk by chunk as matrix products
 *     (same section: state space duality recasts the scan as hardware-
 *     efficient matrix multiplication; chunk length 128 in the feasibility
 *     report, sections 1.4 and 2.6);
 *   - the single-token decode update of the same recurrence;
 *   - entry points built from these: the prefill layer in one call (conv,
 *     then scan), ragged prefill over packed sequences (cu_seqlens), the
 *     decode step in one kernel (cache roll, conv, update), the scan's
 *     backward pass (gradients for training), and the whole Mamba-2 mixer
 *     (in_proj, the path, gated RMSNorm, out_proj) with its linear layers.
 * Discretisation (the pages leave it open; this is the Mamba-2 reading):
 *   dt = softplus(dt_raw + dt_bias), Abar = exp(dt * A), Bbar = dt * B.
 *
 * Notation: b batch, L tokens, H heads, P head dim, N state size (d_state),
 * G groups of B/C (head h uses group h / (H / G)), Q chunk length,
 * k conv width, conv_dim = H*P + 2*G*N.
 *
 * Conventions shared by every call:
 *   - Every tensor argument is a DEVICE pointer owned by the caller.  The
 *     library never allocates or frees device memory, never synchronises the
 *     device or the stream, and keeps no mutable global state (the one
 *     exception, ssd_chunk_scan_fwd_static, says so); calls are thread-safe.
 *     All work is enqueued on `stream` (0 = legacy default).
 *   - I/O tensors (xBC, x, B, C, dt_raw, y, conv_state) have the element
 *     type given by `dtype`; parameters (w, bias, A, D, dt_bias) and SSM
 *     states are float32.  Accumulation is float32; bf16 outputs are
 *     rounded to nearest even.
 *   - Tensors are dense row-major in the layouts stated below, except where
 *     a row stride is taken.  Pointers must be 16-byte aligned and inner
 *     sizes must allow 16-byte vector access where stated.
 *   - Return value: SSD_OK when the work was enqueued;
 *     SSD_ERR_INVALID_ARG for a NULL required pointer, a negative or
 *     inconsistent size, a misaligned pointer or stride, or overlapping
 *     input/output buffers -- nothing is launched;
 *     SSD_ERR_UNSUPPORTED for a valid combination this build has no kernel
 *     for -- nothing is launched;
 *     SSD_ERR_CUDA when a launch failed (cudaGetLastError was not
 *     cudaSuccess; the error is cleared).  Asynchronous faults surface at the
 *     caller's next synchronisation, as for any CUDA work.
 *   - Empty work (b == 0 or L == 0) returns SSD_OK and launches no kernel;
 *     the token tensors are then never touched and may be NULL.  The
 *     exceptions write what a sequence of no tokens still defines:
 *     ssd_chunk_scan_fwd and ssd_conv_scan_fwd with b > 0, L == 0 and a
 *     final_state enqueue a copy of init_state (or zeros) into final_state;
 *     ssd_chunk_scan_fwd_varlen with empty sequences writes their final
 *     states; ssd_chunk_scan_bwd zeroes dA, dD and ddt_bias and copies
 *     dfinal (or zeros) into dinit.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSD_ABI_VERSION 1

/* Entry points are the library's only exported symbols. */
#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,
    SSD_ERR_UNSUPPORTED = 2,
    SSD_ERR_CUDA = 3,
    SSD_ERR_TIMEOUT = 4
} ssd_status_t;

typedef enum ssd_dtype {
    SSD_F32 = 0,
    SSD_BF16 = 1
} ssd_dtype_t;

/* Human-readable name of a status code (static storage; never NULL). */
SSD_API const char* ssd_status_string(ssd_status_t status);

/* SSD_ABI_VERSION of the loaded library. */
SSD_API int ssd_abi_version(void);

/*
 * Causal depthwise conv1d + SiLU.
 *
 *   u[t][c] = SiLU(bias[c] + sum_{j<k} w[c][j] * e[t-k+1+j][c])
 *
 * where e[tau] = xBC[tau] for tau >= 0 and, for tau < 0, the cached input
 * conv_state[c][tau+k] (or 0 when conv_state is NULL).
 *
 *   xBC        [b][L][conv_dim]  dtype, read only
 *   out        [b][L][conv_dim]  dtype, written; must not overlap xBC
 *   w          [conv_dim][k]     float32 taps; tap k-1 multiplies token t
 *   bias       [conv_dim]        float32, may be NULL (zero)
 *   conv_state [b][conv_dim][k]  dtype, may be NULL.  On entry column j holds
 *                                the input at time j-k before this call's
 *                                first token; on exit it holds the last k
 *                                inputs of (old cache | xBC), oldest first.
 *                                With L == 1 this is the decode-step roll.
 * Requirements: 2 <= k <= 4 (else SSD_ERR_UNSUPPORTED); conv_dim a multiple
 * of 8 (bf16) or 4 (f32); xBC, out, w, conv_state 16-byte aligned.
 */
SSD_API ssd_status_t ssd_conv1d_silu(const void* xBC, void* out, const float* w,
                             const float* bias, void* conv_state, int b, int L,
                             int conv_dim, int k, ssd_dtype_t dtype,
                             cudaStream_t stream);

/*
 * Bytes of device workspace ssd_chunk_scan_fwd needs for these sizes
 * (0 when none).  Pure host function; depends only on its arguments and
 * the device properties of the current device.
 */
SSD_API size_t ssd_chunk_scan_workspace_bytes(int b, int L, int H, int P, int N, int G,
                                      int Q, ssd_dtype_t dtype);

/*
 * Chunked SSD scan (prefill).  For every (batch, head), with
 * dt_t = softplus(dt_raw[t] + dt_bias), a_t = dt_t * A:
 *
 *   h_t = exp(a_t) h_{t-1} + dt_t x_t B_t^T        (h: P x N, h_{-1} = init)
 *   y_t = h_t C_t + D x_t
 *
 * evaluated in chunks of Q tokens: intra-chunk (C B^T o L) X with the decay
 * mask L[i][j] = exp(cum_i - cum_j) dt_j (j <= i), chunk states, inter-chunk
 * state passing and the C . h_prev term.  The result does not depend on Q
 * beyond rounding.
 *
 *   x          token t, head h, p at x[(b*L + t)*row_stride + h*P + p]
 *   B, C       token t, group g, n at B[(b*L + t)*row_stride + g*N + n]
 *              (x, B, C may be the three channel ranges of the conv output,
 *              row_stride = conv_dim)                         dtype, read only
 *   dt_raw     [b][L][H]          dtype
 *   dt_bias    [H]                float32, may be NULL (zero)
 *   A          [H]                float32, expected <= 0 (a decaying state)
 *   D          [H]                float32, may be NULL (zero)
 *   init_state [b][H][P][N]       float32, may be NULL (zero state)
 *   y          [b][L][H][P]       dtype, written; must not overlap inputs
 *   final_state[b][H][P][N]       float32, may be NULL; may alias init_state
 *   workspace  device scratch of at least ssd_chunk_scan_workspace_bytes()
 *              bytes (may be NULL when that is 0); contents on entry are
 *              ignored; only this call uses it while it runs
 *   status     optional device int32: set to SSD_ERR_TIMEOUT by the kernels
 *              if a bounded wait gave up (the results are then invalid);
 *              never cleared by the library.  With status NULL a wait that
 *              gave up goes unreported: callers that cannot rule out long
 *              stalls (a GPU shared with other work, the tensor-core path's
 *              cross-CTA hand-offs) should pass one and check it
 * Requirements: P a multiple of 8, N a multiple of 8, H % G == 0, Q in
 * {64, 128}; row_stride a multiple of 8 elements (16 bytes); all pointers
 * 16-byte aligned.
 */
SSD_API ssd_status_t ssd_chunk_scan_fwd(const void* x, const void* B, const void* C,
                                int64_t row_stride, const void* dt_raw,
                                const float* dt_bias, const float* A,
                                const float* D, const float* init_state,
                                void* y, float* final_state, int b, int L,
                                int H, int P, int N, int G, int Q,
                                ssd_dtype_t dtype, void* workspace,
                                size_t workspace_bytes, int32_t* status,
                                cudaStream_t stream);

/*
 * ssd_chunk_scan_fwd without a caller-provided workspace, for callers that
 * cannot allocate device memory on their call path (a host framework that
 * owns every device allocation and forbids raw cudaMalloc, a serving loop
 * that must not allocate per request, a runtime with a fixed memory budget).
 * The pages have no counterpart: this is a deployment convenience.
 *
 * Same arguments, semantics and requirements as ssd_chunk_scan_fwd, minus
 * `workspace` / `workspace_bytes`.  The scratch memory comes from a 10 MiB
 * array compiled into the library, which every GPU that loads the library
 * holds until the process exits.  Nothing is allocated.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - A call whose scratch need (ssd_chunk_scan_workspace_bytes) exceeds
 *     10 MiB returns SSD_ERR_UNSUPPORTED and launches nothing.  The
 *     tensor-core scan needs at most (SM count) x 32 KiB plus a small
 *     control block, about 4.6 MiB on a 148-SM B200.
 *   - All calls on a device share the array; the parts that must start at
 *     zero are cleared on the call's stream.  Calls whose executions overlap
 *     on the GPU (unordered streams) race on the array: order them.
 * Unlike the rest of the library, this entry point keeps global state: the
 * array and the cached per-device addresses.
 */
SSD_API ssd_status_t ssd_chunk_scan_fwd_static(const void* x, const void* B, const void* C,
                                       int64_t row_stride, const void* dt_raw,
                                       const float* dt_bias, const float* A,
                                       const float* D, const float* init_state,
                                       void* y, float* final_state, int b, int L,
                                       int H, int P, int N, int G, int Q,
                                       ssd_dtype_t dtype, int32_t* status,
                                       cudaStream_t stream);

/*
 * Ragged prefill: the chunked scan of ssd_chunk_scan_fwd over several
 * sequences of different lengths packed along one token dimension, each
 * sequence from its own initial state ("Mamba-2 layer" serving: a prefill
 * batch of unequal prompts, or a long prompt processed in pieces with the
 * state handed from one call to the next).  Sequence s is the packed tokens
 * cu_seqlens[s] .. cu_seqlens[s+1]-1; no token of one sequence affects
 * another.
 *
 *   x          [T][.]   x[t*row_stride + h*P + p]           dtype
 *   B, C       [T][.]   B[t*row_stride + g*N + n]           dtype
 *   dt_raw     [T][H]                                       dtype
 *   y          [T][H][P]                                    dtype, written
 *   cu_seqlens [nseq+1] int32, DEVICE memory: cu_seqlens[0] = 0,
 *              non-decreasing, cu_seqlens[nseq] = T.  It is read on the
 *              device: if it breaks these rules, nothing is written and
 *              SSD_ERR_INVALID_ARG is stored in *status.
 *   init_state [nseq][H][P][N] float32 or NULL (zeros)
 *   final_state[nseq][H][P][N] float32 or NULL; an empty sequence's final
 *              state is its initial state (or zero)
 *   status     device int32, REQUIRED (cu_seqlens errors and SSD_ERR_TIMEOUT
 *              are reported there); the caller zeroes it before the call
 *   workspace  ssd_chunk_scan_varlen_workspace_bytes(...) bytes, device,
 *              caller-owned, no initial contents required
 * Other arguments and requirements as for ssd_chunk_scan_fwd.  nseq = 0
 * requires T = 0 and does nothing.
 */
SSD_API size_t ssd_chunk_scan_varlen_workspace_bytes(int nseq, int T, int H, int P, int N, int G,
                                                     int Q, ssd_dtype_t dtype);

SSD_API ssd_status_t ssd_chunk_scan_fwd_varlen(const void* x, const void* B, const void* C,
                                               int64_t row_stride, const void* dt_raw,
                                               const float* dt_bias, const float* A,
                                               const float* D, const float* init_state,
                                               void* y, float* final_state,
                                               const int32_t* cu_seqlens, int nseq, int T,
                                               int H, int P, int N, int G, int Q,
                                               ssd_dtype_t dtype, void* workspace,
                                               size_t workspace_bytes, int32_t* status,
                                               cudaStream_t stream);

/*
 * The prefill layer in one call: ssd_conv1d_silu, then ssd_chunk_scan_fwd on
 * its output (in the Mamba-2 layer the conv, width 4 with SiLU, feeds the
 * scan directly: Nemotron feasibility report, section 1.4; the conv cache of
 * "Hybrid Architectures for Language Models", summary page, appendix C).
 * The conv output goes to the caller's workspace; the results are those of
 * the two calls, bit for bit.
 *
 *   xBC        [b][L][conv_dim]   dtype, conv_dim = H*P + 2*G*N, channels
 *                                 x | B | C; read only
 *   w, bias, conv_state           as for ssd_conv1d_silu (conv_state, if
 *                                 given, is read and rewritten in place)
 *   dt_raw, dt_bias, A, D, init_state, y, final_state, status
 *                                 as for ssd_chunk_scan_fwd
 *   workspace  at least ssd_conv_scan_workspace_bytes(...) bytes of device
 *              scratch (the conv output, b*L*conv_dim elements, then the
 *              scan's workspace), caller-owned, no initial contents required
 * Requirements: those of both calls; no output may overlap an input or the
 * workspace.
 */
SSD_API size_t ssd_conv_scan_workspace_bytes(int b, int L, int H, int P, int N, int G, int Q,
                                             int k, ssd_dtype_t dtype);

SSD_API ssd_status_t ssd_conv_scan_fwd(const void* xBC, const float* w, const float* bias,
                                       void* conv_state, const void* dt_raw,
                                       const float* dt_bias, const float* A, const float* D,
                                       const float* init_state, void* y, float* final_state,
                                       int b, int L, int H, int P, int N, int G, int Q, int k,
                                       ssd_dtype_t dtype, void* workspace,
                                       size_t workspace_bytes, int32_t* status,
                                       cudaStream_t stream);

/*
 * Single-token decode update, in place on the float32 state:
 *
 *   dt = softplus(dt_raw + dt_bias); h <- exp(dt*A) h + dt x B^T;
 *   y = h C + D x
 *
 *   state   [b][H][P][N]  float32, read and rewritten in place
 *   x       [b][.][H][P]  x[bi*row_stride + h*P + p]        dtype
 *   B, C    [b][.][G][N]  B[bi*row_stride + g*N + n]        dtype
 *           (row_stride = conv_dim when reading the conv output)
 *   dt_raw  [b][H]        dtype
 *   dt_bias [H], A [H], D [H]  float32 (dt_bias and D may be NULL)
 *   y       [b][H][P]     dtype, written
 * Requirements: N a multiple of 4 with N <= 256; P >= 1; H % G == 0;
 * state 16-byte aligned.
 */
SSD_API ssd_status_t ssd_state_update(float* state, const void* x, const void* B,
                              const void* C, int64_t row_stride,
                              const void* dt_raw, const float* dt_bias,
                              const float* A, const float* D, void* y, int b,
                              int H, int P, int N, int G, ssd_dtype_t dtype,
                              cudaStream_t stream);

/*
 * The decode step of the layer in one kernel: ssd_conv1d_silu with L = 1 and
 * a cache (roll the cache, convolve the new token, SiLU), then
 * ssd_state_update on its output (the Mamba cache of "Hybrid Architectures
 * for Language Models", summary page, appendix C: the conv cache and the
 * state are the per-layer decode state).  The conv outputs never leave the
 * chip; the results equal those of the two calls bit for bit.
 *
 *   state      [b][H][P][N]       float32, read and rewritten in place
 *   conv_state [b][conv_dim][k]   dtype, REQUIRED, rolled in place (as for
 *                                 ssd_conv1d_silu), conv_dim = H*P + 2*G*N
 *   xBC        [b][conv_dim]      dtype, the new token's x | B | C inputs
 *   w [conv_dim][k], bias [conv_dim] (may be NULL)   float32
 *   dt_raw [b][H] dtype; dt_bias [H], A [H], D [H] float32 (dt_bias, D may be NULL)
 *   y          [b][H][P]          dtype, written
 * One CTA per (sequence, group) convolves the group's B and C channels once
 * and the x channels of its H/G heads, then updates those heads' states.
 * Requirements: 2 <= k <= 4 and N a multiple of 4 with N <= 256 (else
 * SSD_ERR_UNSUPPORTED); H % G == 0; state 16-byte aligned; no buffer may
 * overlap another.
 */
SSD_API ssd_status_t ssd_decode_step(float* state, void* conv_state, const void* xBC, const float* w,
                                     const float* bias, const void* dt_raw, const float* dt_bias,
                                     const float* A, const float* D, void* y, int b, int H, int P,
                                     int N, int G, int k, ssd_dtype_t dtype, cudaStream_t stream);

/*
 * The same decode step in one kernel with a small workspace, so that it can
 * run one CTA per (sequence, head) and keep HBM as busy as ssd_state_update
 * does: every CTA convolves its head's x channels and its group's B and C
 * channels, and the group's B and C cache columns, which its heads share,
 * are rolled by whichever of the group's CTAs finishes reading them last (an
 * atomic count per (sequence, group); no CTA waits for another).  Same
 * arguments, layouts and results as ssd_decode_step (bit for bit), plus
 *   workspace        int32 [b][G], caller-owned, ZERO before the first call
 *                    on it; every call leaves it zero.  Calls that may run
 *                    at the same time need separate workspaces.
 *   workspace_bytes  at least ssd_decode_step_workspace_bytes(b, G)
 * Errors as ssd_decode_step, SSD_ERR_INVALID_ARG for a NULL, unaligned,
 * short or overlapping workspace, and SSD_ERR_UNSUPPORTED for P > 256.
 */
SSD_API size_t ssd_decode_step_workspace_bytes(int b, int G);
SSD_API ssd_status_t ssd_decode_step_ws(float* state, void* conv_state, const void* xBC, const float* w,
                                        const float* bias, const void* dt_raw, const float* dt_bias,
                                        const float* A, const float* D, void* y, int b, int H, int P,
                                        int N, int G, int k, ssd_dtype_t dtype, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass of the chunked scan: the gradients of a loss
 * Loss(y, final_state) through ssd_chunk_scan_fwd, given dy = dLoss/dy and
 * dfinal = dLoss/d(final_state), for training (the Nemotron feasibility
 * report plans forward and backward tests of the Mamba-2 layer, sections
 * 3.2 and 3.3).  The gradients follow the recurrence h_t = exp(dt_t A)
 * h_{t-1} + dt_t x_t B_t^T, y_t = h_t C_t + D x_t of "Hybrid Architectures for
 * Language Models" (summary page, section 2 Background) with dt =
 * softplus(dt_raw + dt_bias).
 *
 *   x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state
 *                 the forward call's inputs, same layouts (init_state may be
 *                 NULL: zero)
 *   dy            [b][L][H][P]   dtype
 *   dfinal        [b][H][P][N]   float32, may be NULL (zero)
 *   dx            [b][L][H][P]   dtype, written
 *   dB, dC        [b][L][G][N]   dtype, written (summed over each group's heads)
 *   ddt_raw       [b][L][H]      dtype, written
 *   dA, dD, ddt_bias [H]         float32, written (summed over the batch)
 *   dinit         [b][H][P][N]   float32, may be NULL (not wanted)
 *   workspace     ssd_chunk_scan_bwd_workspace_bytes(...) bytes: each chunk's
 *                 entering state and per-head dB, dC (float32), caller-owned
 * float32 arithmetic on the CUDA cores, chunks of 32 tokens in matrix form;
 * deterministic.  Requirements: H % G == 0; the shared memory of one CTA,
 * about 4 (2 P N + 64 P + 160 N + 3.8 K) bytes, within the device limit
 * (else SSD_ERR_UNSUPPORTED; P = 64, N = 128 takes 179 KB); element-aligned
 * I/O pointers; no output may overlap an input or another output.
 */
SSD_API size_t ssd_chunk_scan_bwd_workspace_bytes(int b, int L, int H, int P, int N, int G,
                                                  ssd_dtype_t dtype);

SSD_API ssd_status_t ssd_chunk_scan_bwd(const void* x, const void* B, const void* C,
                                        int64_t row_stride, const void* dt_raw,
                                        const float* dt_bias, const float* A, const float* D,
                                        const float* init_state, const void* dy,
                                        const float* dfinal, void* dx, void* dB, void* dC,
                                        void* ddt_raw, float* dA, float* dD, float* ddt_bias,
                                        float* dinit, int b, int L, int H, int P, int N, int G,
                                        ssd_dtype_t dtype, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

/*
 * Linear layer on the tensor cores, y = x W^T: the Mamba-2 mixer's in_proj
 * and out_proj (Nemotron feasibility report, section 3.3: the projections
 * around the scan are linear layers; section 3.2: the mixer module).
 *
 *   y[m][n] = sum_k x[m][k] * w[n][k]      bf16 operands, float32 accumulation,
 *                                          bf16 result (round to nearest even)
 *   x   [M][ldx]  bf16, row m's K inputs at x[m*ldx .. m*ldx + K)
 *   w   [N][ldw]  bf16, output n's K weights at w[n*ldw ..)
 *   y   [M][ldy]  bf16, written (columns < N); must not overlap x or w
 *   status        optional device int32, set to SSD_ERR_TIMEOUT if a bounded
 *                 device wait gave up (the result is then invalid)
 * Requirements: N, K, ldx, ldw, ldy multiples of 8 (16-byte rows); all
 * pointers 16-byte aligned.  M == 0 does nothing.
 */
SSD_API ssd_status_t ssd_linear_bf16(const void* x, int64_t ldx, const void* w, int64_t ldw, void* y,
                                     int64_t ldy, int M, int N, int K, int32_t* status,
                                     cudaStream_t stream);

/*
 * The Mamba-2 mixer forward in one call: in_proj, the hot path (conv1d +
 * SiLU, chunked scan), the gated RMSNorm and out_proj (the block of the
 * Nemotron feasibility report, section 3.2, computes x + Mamba2(RMSNorm(x));
 * this is the Mamba2(.) part).  The pages fix neither the order of in_proj's
 * outputs nor the gate; this follows the readings also taken by the oracle:
 *
 *   zxbcdt = hidden W_in^T, rows of W_in: z (H*P) | xBC (H*P + 2*G*N) | dt_raw (H)
 *   u      = conv1d + SiLU of xBC (as ssd_conv1d_silu, conv_state rolled in place)
 *   y      = the chunked scan of u's x | B | C with dt_raw (as ssd_chunk_scan_fwd)
 *   g      = y * SiLU(z); n = g / sqrt(mean(g^2) + eps) * norm_w, the mean taken
 *            over each of norm_groups equal slices of a token's H*P vector
 *   out    = n W_out^T
 *
 *   hidden  [b][L][d_model] bf16     W_in [2*H*P + 2*G*N + H][d_model] bf16
 *   conv_w  [conv_dim][k] float32, conv_bias [conv_dim] float32 or NULL
 *   conv_state [b][conv_dim][k] bf16 or NULL (read, then rewritten in place)
 *   dt_bias, A, D [H] float32 (dt_bias, D may be NULL); norm_w [H*P] float32
 *   W_out   [d_model][H*P] bf16
 *   init_state, final_state [b][H][P][N] float32 or NULL (may alias)
 *   out     [b][L][d_model] bf16, written
 *   workspace  ssd_mixer_workspace_bytes(...) bytes of device scratch,
 *              caller-owned, no initial contents required
 *   status  optional device int32 (SSD_ERR_TIMEOUT from a bounded wait)
 * Requirements: dtype SSD_BF16 (else SSD_ERR_UNSUPPORTED); those of
 * ssd_chunk_scan_fwd and ssd_conv1d_silu; d_model and H multiples of 8;
 * (H*P / norm_groups) a multiple of 8; eps >= 0; no output may overlap an
 * input or the workspace.  b == 0 or L == 0 writes only final_state (the
 * initial state, or zeros) and leaves conv_state unchanged.
 */
SSD_API size_t ssd_mixer_workspace_bytes(int b, int L, int d_model, int H, int P, int N, int G, int Q,
                                         int k, ssd_dtype_t dtype);

SSD_API ssd_status_t ssd_mixer_fwd(const void* hidden, const void* W_in, const float* conv_w,
                                   const float* conv_bias, void* conv_state, const float* dt_bias,
                                   const float* A, const float* D, const float* norm_w, const void* W_out,
                                   const float* init_state, void* out, float* final_state, int b, int L,
                                   int d_model, int H, int P, int N, int G, int Q, int k, int norm_groups,
                                   float eps, ssd_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                   int32_t* status, cudaStream_t stream);

/*
 * Self-test of the bounded device waits (failure detection without a fault).
 * Every wait of the tensor-core scan gives up after a time limit, records
 * SSD_ERR_TIMEOUT in the call's status word and lets the kernel run to its
 * end, so that a lost arrival never hangs the GPU.  This call launches one
 * thread that waits, through the same wait routine, on a barrier nothing
 * arrives on, for limit_ns nanoseconds.
 *
 *   status    device int32, written: SSD_ERR_TIMEOUT (4) when the wait ran
 *             out as designed; SSD_ERR_CUDA (3) if the routine misbehaved
 *             (returned early, or waited again after giving up).  The caller
 *             zeroes it before the call and reads it after synchronising.
 *   limit_ns  1 .. 1e9 (else SSD_ERR_INVALID_ARG)
 * Returns SSD_OK when the kernel was launched; the context stays usable.
 */
SSD_API ssd_status_t ssd_selftest_bounded_wait(int32_t* status, uint64_t limit_ns,
                                               cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
