// probe.cu -- a diagnostic launch that drives the library's bounded
// mbarrier wait into its timeout on purpose, so that the failure path every
// kernel relies on (error word, CTA abort flag, early return, TMEM release)
// can be checked on a GPU without faulting or hanging it.
//
// One CTA of two warps. Thread 0 waits on an mbarrier that no thread ever
// arrives on, with the caller's time limit: the wait gives up, records
// (timeout, site 1) in the probe's error word and raises the CTA's abort
// flag. Thread 32 waits on a second such mbarrier with the kernels' default
// limit; it must end early, through the abort flag, without recording
// anything. Warp 1 holds 32 TMEM columns across both waits and frees them
// afterwards, as the kernels do on their abort path.
#include <cuda_runtime.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {
namespace {

__device__ unsigned g_probe_err;

__global__ void __launch_bounds__(64, 1) wait_probe_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (threadIdx.x == 0)
        mbar_wait(&bars[0], 0, abort_flag, &g_probe_err, 1, limit_ns);   // never completes
    else if (threadIdx.x == 32)
        mbar_wait(&bars[1], 0, abort_flag, &g_probe_err, 2);             // ends through the abort flag
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }
}

}  // namespace

cudaError_t launch_wait_probe(unsigned long long limit_ns, cudaStream_t s) {
    wait_probe_kernel<<<1, 64, 0, s>>>(limit_ns);
    return cudaGetLastError();
}

unsigned read_clear_probe_error() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_probe_err, sizeof v) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_probe_err, &zero, sizeof zero);
    return v;
}

}  // namespace sage
