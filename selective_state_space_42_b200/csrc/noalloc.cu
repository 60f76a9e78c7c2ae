// noalloc.cu -- selscan_fwd_noalloc: the selective scan with its chunk
// workspace taken from a fixed device array instead of being allocated.
//
// Some callers cannot allocate device memory while they run: code whose whole
// device memory is handed out by another allocator (a framework's caching
// allocator, a fixed arena reserved at start-up), latency-critical loops where
// an allocation may block or fail at the worst moment, and processes where
// stream-ordered memory pools are unavailable or switched off. This entry
// point computes exactly what selscan_fwd computes with the same launch plan,
// but when that plan is chunked its workspace is the file-scope array below,
// which every GPU that loads the library holds until the process exits.
//
// Host code must not use the array's name as a device address: in host code
// it names a host-side stand-in. Every call that needs the workspace looks the
// device address up with cudaGetSymbolAddress (on the current device, which is
// the one the call runs on), checks the result and passes it to the kernels as
// a plain pointer. Nothing is cached: after a device reset, or after the
// primary context is released and created again, the library's module is
// loaded again and the array may sit at a new address, which a kept pointer
// would miss.
#include <cuda_runtime.h>
#include <stdint.h>

#include "selscan.h"
#include "selscan_device.cuh"

namespace {

constexpr size_t kScratchFloats = (size_t)SELSCAN_NOALLOC_WORKSPACE_BYTES / sizeof(float);

// The shared scratch: the plan's workspace (tickets and completion flags,
// which each call zeroes on its stream before its kernels run; chunk
// aggregates and handed-over states, which each call writes before reading).
// It keeps the last call's contents.
static __device__ __align__(256) float g_scratch[kScratchFloats];

// Device address of g_scratch in the current context (looked up afresh on
// every call, see above).
cudaError_t scratch_address(float **out) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_scratch);
    if (e != cudaSuccess) return e;
    if (ptr == nullptr) return cudaErrorInvalidSymbol;
    *out = static_cast<float *>(ptr);
    return cudaSuccess;
}

}  // namespace

extern "C" int selscan_fwd_noalloc(const void *x, const void *delta, const float *A,
                                   const void *B, const void *C, const float *D,
                                   const void *z, const float *delta_bias,
                                   int softplus_flag, void *y, float *final_state,
                                   int64_t batch, int64_t seqlen, int64_t dim,
                                   int64_t dstate, selscan_dtype_t dtype,
                                   selscan_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    selscan::FwdPlan plan;
    bool done = false;
    const int st = selscan::fwd_setup(x, delta, A, B, C, D, z, delta_bias, softplus_flag,
                                      nullptr, nullptr, nullptr, nullptr, 0, 0, y, final_state, batch, seqlen, dim, dstate, dtype,
                                      stream, &plan, &done);
    if (st != SELSCAN_OK || done) return st;
    if (plan.ws_bytes > (size_t)SELSCAN_NOALLOC_WORKSPACE_BYTES) return SELSCAN_ERR_WORKSPACE;
    float *scratch = nullptr;
    if (plan.ws_bytes > 0) {
        cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return selscan::cuda_fail(e);
    }
    cudaError_t e = selscan::fwd_run(&plan, scratch, stream);
    return e == cudaSuccess ? SELSCAN_OK : selscan::cuda_fail(e);
}
