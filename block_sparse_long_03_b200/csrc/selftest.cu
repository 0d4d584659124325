// selftest.cu -- a check of the failure path shared by the tensor-core
// kernels: a bounded mbarrier wait that is never satisfied gives up after its
// limit, records MSA_ERR_DEVICE_TIMEOUT in the error word, and the kernel
// frees its TMEM and returns, leaving the context usable.  Nothing faults,
// traps or spins without a bound.
#include "tc.cuh"

namespace msa {
namespace {

__global__ void wait_timeout_kernel(uint32_t *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x / 32;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);                  // one arrival expected; none comes
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&tmem_slot, 32);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (threadIdx.x == 32) tc::mbar_wait(&bar, 0, err, (volatile int *)&abort_flag, limit_ns);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem_slot, 32);
    }
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                                 uint32_t limit_us, void *stream) {
    if (!workspace || ((uintptr_t)workspace % 256) != 0 || workspace_bytes < msa::kErrorBytes)
        return MSA_ERR_WORKSPACE;
    if (limit_us == 0 || limit_us > 1000000) return MSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t *err = (uint32_t *)workspace;
    cudaError_t e = cudaMemsetAsync(err, 0, msa::kErrorBytes, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    msa::wait_timeout_kernel<<<1, 64, 0, st>>>(err, (uint64_t)limit_us * 1000ull);
    msa::count_launches(1);
    return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
