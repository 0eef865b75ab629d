// selftest.cu -- exercises the failure path every pipeline wait shares.
//
// Each kernel waits on mbarrier phases with mbar_wait (ptx.cuh): a bounded
// spin that, once its wall-clock limit (1 s, %globaltimer) has passed, ORs
// ATTN_DEVERR_TIMEOUT into the caller's error word and returns false so the
// kernel can unwind.  This kernel makes such a wait run out on purpose -- on
// a barrier phase that nothing completes -- so a test can check the status
// word and that the context stays usable afterwards.  No fault, no trap, no
// unbounded spin.
//
// A second kernel evaluates the prefill softmax's FMA-pipe exponential
// (exp2_poly2, softmax_math.cuh) on given inputs, so a test can hold the
// device's results against 2^x and the stated error bound.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/attn.h"
#include "ptx.cuh"
#include "softmax_math.cuh"

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

// y[i] = exp2_poly2(x[i]) for i < n; pairs (x[2k], x[2k+1]) go through one
// call, an odd last element is paired with 0.
__global__ void exp2_poly_selftest_kernel(const float *x, float *y, int n) {
    const int pairs = (n + 1) / 2;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < pairs; k += gridDim.x * blockDim.x) {
        const int i = 2 * k;
        const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
        float r0, r1;
        f2_unpack(exp2_poly2(f2_pack(a, b)), r0, r1);
        y[i] = r0;
        if (i + 1 < n) y[i + 1] = r1;
    }
}

}  // namespace

attn_status launch_exp2_poly_selftest(const float *x, float *y, int n, cudaStream_t stream) {
    if (n == 0) return ATTN_OK;
    const int pairs = (n + 1) / 2;
    const int grid = (pairs + 255) / 256 < 4096 ? (pairs + 255) / 256 : 4096;
    exp2_poly_selftest_kernel<<<grid, 256, 0, stream>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

attn_status launch_wait_timeout_selftest(int32_t *err_flag, int32_t *result, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err_flag, result);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
