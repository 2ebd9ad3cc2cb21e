// scan_block4_noalloc: scan_block4 with its scratch in a fixed block of
// device memory that belongs to the library, for callers that must not
// allocate device memory themselves.
//
// Who needs this: code that runs where its own allocator owns every byte of
// device memory (a serving process that reserved the whole GPU up front, an
// embedded runtime with a fixed arena), code that may not call cudaMalloc
// because cudaMalloc can synchronise the device and stall other streams, and
// plugins or callbacks that only receive input and output pointers.  They
// cannot size and pass a workspace, so this entry point brings its own.
//
// The scratch is one file-scope __device__ array.  Every GPU that loads the
// library holds it until the process exits, and all calls on a device share
// it: calls that overlap on that GPU (other streams, other host threads)
// race on it and must be serialised by the caller.  The scan's ticket
// counter and flag words are cleared on the stream at the start of every
// call; the rest is overwritten before it is read.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "launchers.h"

static __device__ __align__(256) unsigned char g_scan_scratch[SLSTM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Per device: the context the address was looked up in, and the address.
// A device reset ends that context; the next call runs in a new one and
// looks the address up again.
struct ScratchEntry {
    CUcontext ctx;
    void *ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 ctx_getter()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    }
    return fn;
}

// Device address of g_scan_scratch in the current device's current context,
// looked up once per device and context (the host-side name of the array is
// only a stand-in for it).
cudaError_t scratch_on_current_device(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    auto get_ctx = ctx_getter();
    if (get_ctx == nullptr) return cudaErrorInitializationError;
    // null before the runtime has made this device's context current here
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
    std::lock_guard<std::mutex> lock(g_mutex);
    ScratchEntry &s = g_scratch[dev];
    if (ctx == nullptr || s.ptr == nullptr || s.ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scan_scratch);   // also initialises the context when needed
        if (e != cudaSuccess) return e;
        if (ctx == nullptr && (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return cudaErrorInitializationError;
        s.ctx = ctx;
        s.ptr = p;
    }
    *out = s.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" int scan_block4_noalloc(const float *A, const float *b, const float *y0, float *y, int B,
                                   int T, int d, int flags, slstm_stream_t stream)
{
    if ((flags & ~SLSTM_SCAN_REVERSE_T) != 0) return SLSTM_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || d < 1) return SLSTM_ERR_INVALID_ARG;
    const size_t need = slstm_workspace_size(SLSTM_OP_SCAN_BLOCK4, B, T, 0, d);
    if (need == 0) return SLSTM_ERR_INVALID_ARG;
    if (need > (size_t)SLSTM_NOALLOC_SCRATCH_BYTES) return SLSTM_ERR_UNSUPPORTED;
    const uintptr_t mask = 15u;
    if (!A || !b || !y || (reinterpret_cast<uintptr_t>(A) & mask) || (reinterpret_cast<uintptr_t>(b) & mask) ||
        (reinterpret_cast<uintptr_t>(y) & mask) || (y0 && (reinterpret_cast<uintptr_t>(y0) & mask)))
        return SLSTM_ERR_INVALID_ARG;
    if (y == A || y == b) return SLSTM_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return SLSTM_ERR_CUDA;
    const cudaError_t e = slstm::scan_block4_launch(A, b, y0, y, B, T, d, (flags & SLSTM_SCAN_REVERSE_T) != 0,
                                                    scratch, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SLSTM_OK : SLSTM_ERR_CUDA;
}
