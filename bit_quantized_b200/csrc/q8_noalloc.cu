// q8_linear_int8_mixed_noalloc: the LLM.int8 mixed-decomposition linear for
// callers that cannot allocate device memory.
//
// q8_linear_int8_mixed needs a scratch workspace (the outlier mask and column
// list, the int8 codes of the regular stream, and the gathered fp16 outlier
// columns).  Some callers have no way to provide one: an inference engine that
// plans all of its device memory ahead of time and forbids allocation while it
// serves requests, a plain C caller without a device allocator of its own, or
// code that runs where calling cudaMalloc is not allowed.  For them this file
// keeps one fixed scratch buffer in the library itself, as a static device
// array, and runs the same kernels on it.
//
// The buffer is a file-scope __device__ array.  In host code its name is only
// a stand-in for the device object, not a device address, so the address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device, and cached.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "q8_internal.h"

namespace {

// Bytes of the library-owned scratch (Q8_NOALLOC_SCRATCH_BYTES, 64 MiB):
// enough for, e.g., m = 512 tokens with n = k = 4096, since the workspace
// holds every column as a potential outlier.
constexpr size_t kScratchBytes = Q8_NOALLOC_SCRATCH_BYTES;
// Size limits of q8_linear_int8_mixed (M, N <= 2^31 - 1; K <= 32768 for the
// INT32 accumulator).
constexpr int64_t kMaxDimNoalloc = (int64_t(1) << 31) - 1;
constexpr int64_t kMaxKInt8Noalloc = 32768;

// Shared by every call on a device and kept until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's scratch; looked up on the first call made
// on the device (with that device current) and cached for later calls.  A
// cudaDeviceReset destroys the array with the context, so the cached address
// is only valid until the device is reset (documented in include/q8.h).
q8_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return Q8_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return Q8_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return Q8_OK;
}

}  // namespace

extern "C" {

q8_status q8_linear_int8_mixed_noalloc(const void* X, q8_dtype x_dtype, int64_t m, int64_t k,
                                       int64_t ldx, const q8_weight* w, const void* W16,
                                       float threshold, const float* bias, void* Y, int64_t ldy,
                                       uint8_t* outlier_mask, int32_t* outlier_count,
                                       int32_t* acc_debug, float* y16_debug,
                                       q8_stream_t stream) {
    if (!w) return Q8_ERR_NULL;
    // The sizes the scratch is computed from must be valid ones first (the
    // same limits q8_linear_int8_mixed applies), then the scratch must fit.
    if (m < 0 || m > kMaxDimNoalloc || w->n < 0 || w->n > kMaxDimNoalloc || k <= 0 ||
        k != w->k || k > kMaxKInt8Noalloc)
        return Q8_ERR_SHAPE;
    if (q8_workspace_size(Q8_OP_LINEAR_INT8_MIXED, m, w->n, k) > kScratchBytes) return Q8_ERR_SHAPE;
    void* scratch = nullptr;
    const q8_status st = scratch_address(&scratch);
    if (st != Q8_OK) return st;
    // Every region of the scratch is written by the kernels before it is read
    // (mask, column list and count by the outlier pass, codes/scales/row sums
    // by the row pass, the fp16 outlier columns with their zero padding by the
    // gathers), so nothing has to be cleared between calls.
    return q8_linear_int8_mixed(X, x_dtype, m, k, ldx, w, W16, threshold, bias, Y, ldy,
                                outlier_mask, outlier_count, acc_debug, y16_debug, scratch,
                                kScratchBytes, stream);
}

}  // extern "C"
