// rb_gemv_noalloc: the batch-1..64 matvec for callers that cannot allocate
// device memory. Its scratch (the work counters and K-split partial sums that
// rb_gemv keeps in a caller-provided workspace) lives in one static device
// array per GPU instead, so the call itself allocates nothing.
#include "../../include/rb_api.h"
#include "rb_internal.cuh"

#include <cstdio>
#include <mutex>

namespace rb {
void set_error_message(const char* msg);
}

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoallocScratchBytes = size_t(1) << 20;   // 1 MiB
__device__ __align__(256) unsigned char rb_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

}  // namespace

namespace rb {

// The device address of the array on the current device. In host code the
// symbol is only a host-side stand-in, so it is looked up once per device,
// with that device current, and cached. rb_gemv_check(NULL, ...) reads the
// error word of the array through this address too.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, rb_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return cudaSuccess;
}

}  // namespace rb

extern "C" rb_status rb_gemv_noalloc(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype,
                                     rb_layout L, const void* x, int64_t ldx, int32_t T,
                                     void* y, rb_dtype y_dtype, int64_t ldy, void* stream) {
    // size first: a request that does not fit is refused before any CUDA call
    const size_t need = rb_gemv_workspace_bytes(L, T);
    if (need > kNoallocScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "rb_gemv_noalloc: this shape needs %zu bytes of scratch, the static array holds %zu; "
                 "use rb_gemv with a workspace", need, kNoallocScratchBytes);
        rb::set_error_message(msg);
        return RB_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    const cudaError_t e = rb::noalloc_scratch(&scratch);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof(msg), "rb_gemv_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        rb::set_error_message(msg);
        return RB_ERR_CUDA;
    }
    // rb_gemv validates the arguments and launches (the static scratch starts
    // at zero and every call leaves its counters at zero); an invalid layout
    // (need == 0) is reported by it as well
    return rb_gemv(planes, alpha, alpha_dtype, L, x, ldx, T, y, y_dtype, ldy, scratch, kNoallocScratchBytes,
                   stream);
}
