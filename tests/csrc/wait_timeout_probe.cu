// Test-only kernel: exercises the library's bounded mbarrier wait (titans_long_term_b200/csrc/ptx.cuh)
// on a barrier that nothing ever arrives on. The wait must give up after its time limit and the
// kernel must record the timeout in a status word and return, leaving the context usable.
#include <cuda_runtime.h>

#include "../../titans_long_term_b200/csrc/ptx.cuh"

using namespace titans;

__global__ void never_arrives(unsigned* status, unsigned long long* waited_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer_ns();
        const bool ok = mbar_wait(&bar, 0);  // phase 0 never completes
        *waited_ns = globaltimer_ns() - t0;
        if (!ok) atomicOr(status, kStatusTimeoutMma);
    }
}

extern "C" int run_never_arrives(unsigned* status_host, unsigned long long* waited_ns_host) {
    unsigned* st = nullptr;
    unsigned long long* ns = nullptr;
    if (cudaMalloc(&st, sizeof(unsigned)) != cudaSuccess) return 1;
    if (cudaMalloc(&ns, sizeof(unsigned long long)) != cudaSuccess) return 2;
    cudaMemset(st, 0, sizeof(unsigned));
    never_arrives<<<1, 32>>>(st, ns);
    cudaError_t e = cudaDeviceSynchronize();
    cudaMemcpy(status_host, st, sizeof(unsigned), cudaMemcpyDeviceToHost);
    cudaMemcpy(waited_ns_host, ns, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
    cudaFree(st);
    cudaFree(ns);
    return e == cudaSuccess ? 0 : 3;
}
