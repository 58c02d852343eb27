// noalloc.cu -- a Newton forward entry point that allocates nothing.
//
// Some callers cannot allocate device memory when they want to run the
// forward: a host framework that owns every device allocation through its own
// pool and forbids direct cudaMalloc, a latency-bound loop that cannot afford
// the implicit synchronisation of cudaMalloc/cudaFree, or a deployment whose
// device-memory budget is fixed at start-up.  For them this entry point runs
// the same forward kernels with their scratch memory (the workspace of
// pararnn_newton_forward) in a fixed array that is part of the library's
// device image.  Every GPU that loads the library holds that array until the
// process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "pararnn_b200.h"

namespace pararnn {
void set_last_error(const char* msg);  // defined in pararnn_abi.cu
}

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB, the largest workspace this entry point serves
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Per device: the array's device address, looked up with that device
// current (in host code the array's name is only a stand-in, not an address
// a kernel may use).  A failed look-up is not remembered, so a later call
// retries it.  The array needs no clearing: every forward call clears the
// part of its workspace that it reads.
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices];

cudaError_t scratch_for(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return e;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" pararnn_status pararnn_newton_forward_noalloc(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                                         pararnn_dtype px_dtype, const void* preacts,
                                                         const float* diag_w, const float* h0, int K, float* H_out,
                                                         float* resid_hist, int wait_status, void* stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        pararnn::set_last_error("pararnn_newton_forward_noalloc: no current CUDA device");
        return PARARNN_ECUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        pararnn::set_last_error("pararnn_newton_forward_noalloc: device ordinal out of range");
        return PARARNN_EINVAL;
    }
    if (K < 0) {
        pararnn::set_last_error("pararnn_newton_forward_noalloc: K must be 0 (the measured K*) or at least 1");
        return PARARNN_EINVAL;
    }
    // 0 means invalid sizes or cell; pararnn_workspace_bytes has then already
    // stored the specific reason for pararnn_last_error()
    const size_t need = pararnn_workspace_bytes(cell, B, T, D, K);
    if (need == 0) return PARARNN_EINVAL;
    if (need > kScratchBytes) {
        pararnn::set_last_error(
            "pararnn_newton_forward_noalloc: this problem needs more scratch memory than the fixed 32 MiB array "
            "holds; use pararnn_newton_forward with a workspace of pararnn_workspace_bytes() bytes");
        return PARARNN_EINVAL;
    }
    void* scratch = nullptr;
    if (scratch_for(dev, &scratch) != cudaSuccess) {
        pararnn::set_last_error("pararnn_newton_forward_noalloc: could not look up the scratch array on this device");
        return PARARNN_ECUDA;
    }
    pararnn_status st = pararnn_newton_forward(cell, B, T, D, px_dtype, preacts, diag_w, h0, K, H_out, scratch,
                                               kScratchBytes, resid_hist, stream);
    if (st != PARARNN_OK || !wait_status) return st;
    return pararnn_status_sync(scratch, stream);
}
