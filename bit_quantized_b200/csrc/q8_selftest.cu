// Self-test of the device-side failure detection.
//
// Every kernel of the library bounds its barrier waits: a wait that runs out
// records Q8_ERR_DEVICE_TIMEOUT in the per-device status word and raises the
// CTA's abort flag; the CTA's other roles see the flag, leave their own waits,
// and the CTA frees its tensor memory and returns instead of hanging.  In a
// correct run no wait ever runs out, so that path would otherwise never
// execute.  wait_timeout_kernel has the GEMM kernels' structure (a producer
// warp, an MMA warp and four epilogue warps sharing one abort flag, TMEM
// allocated for the CTA) and a producer whose barrier nothing ever arrives
// on, with a short wait limit given by the host.  Nothing faults, traps or
// spins without a bound: the kernel ends after about that limit.
#include <cuda_runtime.h>

#include <cstdint>

#include "q8_device.cuh"
#include "q8_internal.h"

namespace q8 {
namespace {

constexpr int kSelfTestThreads = 192;
constexpr uint32_t kSelfTestTmemCols = 32;

__global__ void __launch_bounds__(kSelfTestThreads, 1)
wait_timeout_kernel(uint64_t limit_ns, int* status) {
    __shared__ __align__(8) uint64_t never_bar;   // no thread ever arrives here
    __shared__ __align__(8) uint64_t full_bar;    // the producer would release the MMA role
    __shared__ __align__(8) uint64_t tfull_bar;   // the MMA role would release the epilogue
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x / 32;
    if (threadIdx.x == 0) {
        mbar_init(&never_bar, 1);
        mbar_init(&full_bar, 1);
        mbar_init(&tfull_bar, 1);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, kSelfTestTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    if (warp == 0) {
        // Producer: waits (bounded by limit_ns) for a stage nothing releases;
        // the timeout records the status and raises the abort flag.
        if (elect_one()) {
            if (mbar_wait(&never_bar, 0, &abort_sh, status, limit_ns)) mbar_arrive(&full_bar);
        }
        __syncwarp();
    } else if (warp == 1) {
        // MMA role: waits for the producer; leaves on the abort flag.
        if (elect_one()) {
            if (mbar_wait(&full_bar, 0, &abort_sh, status)) mbar_arrive(&tfull_bar);
        }
        __syncwarp();
    } else {
        // Epilogue warps: every thread waits for the accumulator; all leave on
        // the abort flag.
        mbar_wait(&tfull_bar, 0, &abort_sh, status);
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kSelfTestTmemCols);
    }
}

}  // namespace
}  // namespace q8

using namespace q8;

extern "C" q8_status q8_selftest_wait_timeout(int32_t limit_us, q8_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return Q8_ERR_SHAPE;
    const q8_status st = q8_device_check();
    if (st != Q8_OK) return st;
    int* status = device_status_ptr();
    if (!status) return Q8_ERR_CUDA;
    wait_timeout_kernel<<<1, kSelfTestThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(limit_us) * 1000ull, status);
    if (cudaGetLastError() != cudaSuccess) return Q8_ERR_LAUNCH;
    return Q8_OK;
}
