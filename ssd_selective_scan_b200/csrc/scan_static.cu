// scan_static.cu -- ssd_chunk_scan_fwd_static: the chunked scan for callers
// that cannot allocate device memory.
//
// Some callers cannot allocate device memory on the call path at all: code
// running under a host framework that owns every device allocation through
// its own allocator and forbids raw cudaMalloc, serving loops that must not
// allocate per request (cudaMalloc can synchronise the device and can fail
// under fragmentation), or embedded runtimes with a fixed memory budget set
// up at start.  For them this entry point takes the scan's scratch memory
// from a fixed array compiled into the library instead of from the caller.
//
// The array is kStaticScratchBytes (10 MiB) of file-scope __device__ memory:
// every GPU that loads this library holds it until the process exits.  The
// tensor-core scan needs at most (SM count) x 32 KiB + a small control
// block (about 4.6 MiB on a 148-SM B200), so every call it can serve fits;
// a call whose scratch need (ssd_chunk_scan_workspace_bytes) exceeds the
// array is refused with SSD_ERR_UNSUPPORTED before anything is launched.
//
// In host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, on the first call made on it; later calls reuse the
// cached address.  Because that first call on a device does the look-up (a
// host-side runtime call), make it before any stream capture.  All calls on
// a device share the one array and it keeps
// the last call's contents: the work that must start from zero (the CTA
// ticket counter and hand-off flags) is cleared on the call's stream by the
// scan itself, and everything else is written before it is read.  Two calls
// whose executions overlap on the GPU (different streams, no ordering
// between them) race on the array; callers must order them.
//
// Nothing here allocates: no cudaMalloc, cudaFree or allocating library
// routine is called.
#include <atomic>

#include "ssd.h"

namespace {

constexpr size_t kStaticScratchBytes = 10u << 20;   // 10 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of this device's copy of the array (looked up once per
// device, with the device current).  Returns nullptr and sets *err on error.
void* scratch_for_current_device(cudaError_t* err)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *err = e;
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* q = nullptr;
    e = cudaGetSymbolAddress(&q, g_scan_scratch);
    if (e != cudaSuccess || q == nullptr) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
        return nullptr;
    }
    // threads racing on the first call store the same address
    g_scratch_addr[dev].store(q, std::memory_order_release);
    return q;
}

}  // namespace

extern "C" SSD_API ssd_status_t ssd_chunk_scan_fwd_static(
    const void* x, const void* B, const void* C, int64_t row_stride, const void* dt_raw,
    const float* dt_bias, const float* A, const float* D, const float* init_state, void* y,
    float* final_state, int b, int L, int H, int P, int N, int G, int Q, ssd_dtype_t dtype,
    int32_t* status, cudaStream_t stream)
{
    const size_t need = ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype);
    if (need > kStaticScratchBytes) return SSD_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (need > 0) {
        cudaError_t err = cudaSuccess;
        scratch = scratch_for_current_device(&err);
        if (!scratch) {
            (void)cudaGetLastError();
            return SSD_ERR_CUDA;
        }
    }
    return ssd_chunk_scan_fwd(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y, final_state, b,
                              L, H, P, N, G, Q, dtype, scratch, scratch ? kStaticScratchBytes : 0, status,
                              stream);
}
