// varlen_prep.cu -- device-side preparation of a ragged (cu_seqlens) scan:
// the token offsets live on the device, so the host never reads them.
//
// One CTA, before the scan kernel on the same stream:
//   - zeroes the scan's control block (ticket counter, hand-off flags);
//   - checks cu_seqlens: cu[0] = 0, non-decreasing, cu[nseq] = T.  On
//     failure it sets hdr[0] = 1 (the scan then does nothing) and writes
//     SSD_ERR_INVALID_ARG into the status word;
//   - writes seq_units[s] = H * (chunks of the sequences before s) and
//     hdr[1] = the total (the tensor-core scan's unit list);
//   - writes the final state of every empty sequence: its initial state, or
//     zero.
#include "kernels.h"
#include "ssd.h"

namespace ssd {
namespace {

constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads)
varlen_prep_kernel(const int* __restrict__ cu, int nseq, int T, int H, int Q, int* hdr, int* seq_units,
                   int* ctrl, int ctrl_ints, const float* __restrict__ init_state, float* final_state,
                   long long state_elems, int32_t* status)
{
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = 0;
    __syncthreads();
    for (int i = tid; i < ctrl_ints; i += kPrepThreads) ctrl[i] = 0;
    for (int s = tid; s < nseq; s += kPrepThreads)
        if (cu[s + 1] < cu[s]) bad = 1;
    if (tid == 0 && (cu[0] != 0 || cu[nseq] != T)) bad = 1;
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            hdr[0] = 1;
            hdr[1] = 0;
            if (status) atomicExch(reinterpret_cast<int*>(status), (int)SSD_ERR_INVALID_ARG);
        }
        return;
    }
    if (tid == 0) {
        int acc = 0;
        for (int s = 0; s < nseq; ++s) {
            if (seq_units) seq_units[s] = acc;
            acc += H * ((cu[s + 1] - cu[s] + Q - 1) / Q);
        }
        if (seq_units) seq_units[nseq] = acc;
        hdr[0] = 0;
        hdr[1] = acc;
    }
    if (final_state) {
        for (int s = 0; s < nseq; ++s) {
            if (cu[s + 1] != cu[s]) continue;
            const size_t base = (size_t)s * (size_t)state_elems;
            for (long long e = tid; e < state_elems; e += kPrepThreads)
                final_state[base + e] = init_state ? init_state[base + e] : 0.0f;
        }
    }
}

}  // namespace

cudaError_t launch_varlen_prep(const int* cu_seqlens, int nseq, int T, int H, int Q, int* hdr, int* seq_units,
                               int* ctrl, int ctrl_ints, const float* init_state, float* final_state,
                               long long state_elems_per_seq, int32_t* status, cudaStream_t s)
{
    varlen_prep_kernel<<<1, kPrepThreads, 0, s>>>(cu_seqlens, nseq, T, H, Q, hdr, seq_units, ctrl, ctrl_ints,
                                                  init_state, final_state, state_elems_per_seq, status);
    return cudaGetLastError();
}

}  // namespace ssd
