// dg_sampler_step_noalloc: the sampler step with its scratch memory in a fixed device array.
//
// dg_sampler_step needs a little scratch memory (a counter per row and a 16-byte record per
// 512-id chunk of each row) and asks its caller for it.  Some callers cannot provide it: code
// that runs where allocating is not allowed (a serving loop that must not call cudaMalloc,
// which can synchronize the whole device, on its hot path; an embedding runtime that owns all
// device memory and hands the library only its input and output buffers; a process whose
// memory pool is already fully reserved).  For them this entry point keeps that scratch in a
// file-scope device array of DG_NOALLOC_SCRATCH_BYTES that comes with the library: every GPU on
// which the library is loaded holds the array until the process exits, and no call allocates.
//
// The array's host-side name is only a stand-in for the symbol, not a device address, so the
// device address is looked up with cudaGetSymbolAddress, once per device, with that device
// current, during the first call made on it; make that first call before any stream capture.
// The address is cached per device index for the life of the process: a process that calls
// cudaDeviceReset on a device must not call this entry point on that device afterwards (the
// reset unloads the module, and the cached address would name memory that is gone).  Every call
// shares the one array: two calls that overlap on the GPU (on different streams, or from
// different threads) race and corrupt each other's results.  Each call checks all of its
// arguments first and only then clears the part of the array it uses and launches, so a refused
// call enqueues nothing and the contents left by an earlier call never matter.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/dg.h"
#include "kernels.cuh"

namespace dg {
void set_error_message(int code, const char* msg);
}

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DG_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (looked up on first use).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int dg_sampler_step_noalloc(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t,
                                       int32_t B, int32_t C, int32_t V, int schedule, const double* t,
                                       const double* dt, const float* inv_tau, uint64_t seed, uint32_t step,
                                       int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax,
                                       float* max_prob, float* lse, float* entropy, uint8_t* branch,
                                       dg_stream_t stream) {
    const long long rows = static_cast<long long>(B) * C;
    const bool shaped = B >= 1 && C >= 1 && V >= 1 && rows <= 0x7fffffffLL;
    const size_t need = shaped ? dg_sampler_step_workspace_size(static_cast<int32_t>(rows), V) : 0;
    if (need > static_cast<size_t>(DG_NOALLOC_SCRATCH_BYTES)) {
        char msg[256];
        std::snprintf(msg, sizeof(msg),
                      "B*C = %lld rows of V = %d need %zu bytes of scratch; the fixed array holds %d bytes "
                      "(use dg_sampler_step with a caller workspace)",
                      rows, V, need, DG_NOALLOC_SCRATCH_BYTES);
        dg::set_error_message(DG_ERR_WORKSPACE, msg);
        return DG_ERR_WORKSPACE;
    }
    void* ws = nullptr;
    cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) {
        dg::set_error_message(DG_ERR_CUDA, cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    // Counters must start at zero (the previous call may have used the array with another shape):
    // cleared on the stream after every argument check has passed.
    return dg::sampler_step_impl(logits, logits_dtype, ld, x_t, B, C, V, schedule, t, dt, inv_tau, seed, step,
                                 x0_mode, x_next, x0_hat, argmax, max_prob, lse, entropy, branch, ws,
                                 static_cast<size_t>(DG_NOALLOC_SCRATCH_BYTES), stream, true);
}
