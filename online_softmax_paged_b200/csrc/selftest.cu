// selftest.cu -- exercises the failure path every pipeline wait shares.
//
// Each kernel waits on mbarrier phases with mbar_wait (ptx.cuh): a bounded
// spin that, once its wall-clock limit (1 s, %globaltimer) has passed, ORs
// ATTN_DEVERR_TIMEOUT into the caller's error word and returns false so the
// kernel can unwind.  This kernel makes such a wait run out on purpose -- on
// a barrier phase that nothing completes -- so a test can check the status
// word and that the context stays usable afterwards.  No fault, no trap, no
// unbounded spin.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/attn.h"
#include "ptx.cuh"

namespace osp {
namespace {

__global__ void wait_timeout_selftest_kernel(int32_t *err, int32_t *result) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // one arrival is expected and none is made: phase 0 never completes
    const bool ok = mbar_wait(&bar, 0u, err);
    if (threadIdx.x == 0 && result) *result = ok ? 1 : 0;
}

}  // namespace

attn_status launch_wait_timeout_selftest(int32_t *err_flag, int32_t *result, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err_flag, result);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
