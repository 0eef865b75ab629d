// fp8_quant.cu -- block quantisation of Q or K to e4m3, with optional
// incoherent processing, for the FP8 prefill.
//
// Method (pages): "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
// §二 "FlashAttention-3改进": the forward pass runs its GEMMs on FP8 tensor
// cores, and block quantisation plus incoherent processing limit the accuracy
// lost in the conversion.  Here the QK^T product is the FP8 one.
//
// Persistent CTAs (two per SM), one thread per row of a (head, 128-row
// block); while one block is converted the next block's rows are already in
// flight into the other input buffer.  Per block:
//   y     = x D H                 (rotation: random signs D, Sylvester
//                                  Hadamard H, in-register butterflies; else y = x)
//   amax  = max |y|               (fp32, exact)
//   r     = 448 / amax            (IEEE division; amax = 0: 1; overflow: FLT_MAX)
//   code  = e4m3_rn_satfinite(y * r)
//   scale = amax / (448 sqrt(d))  with rotation, amax / 448 without (in
//                                  double, rounded once to fp32; amax = 0: 1)
// so code * scale approximates the orthogonally rotated row y / sqrt(d) (or
// x), and (Q D H)(K D H)^T / d = Q K^T keeps the attention scores.
// The bf16 block is read with coalesced 16-byte loads into a swizzled shared
// buffer (chunk c of row r at c ^ (r & 15): conflict-free row reads), and the
// codes leave the same way.  The random signs are applied as XOR masks on the
// bf16 bits (kept in shared memory) and the butterflies of stride >= 2 run on
// packed fp32 pairs.  HBM-bound: 2 bytes in, 1 byte out per element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "launch.h"
#include "ptx.cuh"

namespace osp {
namespace {

constexpr int kQRows = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Persistent: CTA c takes blocks c, c + gridDim.x, ...; while one block is
// converted, the next one's bf16 rows are already on their way into the
// other input buffer (cp.async, 16 bytes per copy, swizzled destinations).
template <int D, bool ROT>
__global__ void __launch_bounds__(kQRows, 2) quantize_qk_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                uint8_t *__restrict__ codes,
                                                                float *__restrict__ scales,
                                                                const int8_t *__restrict__ signs, int N, int nblk,
                                                                int total) {
    constexpr int kChunks = D / 8;    // 16-byte chunks of a bf16 row
    constexpr int kCChunks = D / 16;  // 16-byte chunks of a code row
    extern __shared__ __align__(16) uint8_t qsm[];
    uint8_t *in_buf[2] = {qsm, qsm + kQRows * D * 2};
    uint8_t *out_buf = qsm + 2 * kQRows * D * 2;
    __shared__ __align__(16) uint32_t sign_mask[D / 2];  // per bf16x2 word: the sign bits to flip
    __shared__ float warp_max[kQRows / 32];
    const int t = threadIdx.x;

    if (ROT && t < D / 2)
        sign_mask[t] = (__ldg(signs + 2 * t) < 0 ? 0x8000u : 0u) | (__ldg(signs + 2 * t + 1) < 0 ? 0x80000000u : 0u);

    auto issue = [&](int blk, uint8_t *buf) {
        const int bh = blk / nblk, b = blk - bh * nblk;
        const int r0 = b * kQRows, rows = min(kQRows, N - r0);
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x + ((size_t)bh * N + r0) * D);
        const uint32_t sb = smem_u32(buf);
        for (int k = t; k < rows * kChunks; k += kQRows) {
            const int r = k / kChunks, c = k - r * kChunks;
            cp_async16(sb + r * D * 2 + ((c ^ (r & (kChunks - 1))) << 4), src + (size_t)k * 16);
        }
    };

    int it = 0;
    if ((int)blockIdx.x < total) issue(blockIdx.x, in_buf[0]);
    cp_async_commit();
    for (int blk = blockIdx.x; blk < total; blk += gridDim.x, ++it) {
        const uint8_t *buf = in_buf[it & 1];
        if (blk + (int)gridDim.x < total) issue(blk + gridDim.x, in_buf[(it + 1) & 1]);
        cp_async_commit();
        cp_async_wait_prev();  // this block's copies have landed (the next block's may not)
        __syncthreads();

        const int bh = blk / nblk, b = blk - bh * nblk;
        const int r0 = b * kQRows, rows = min(kQRows, N - r0);
        float v[D];
        if (t < rows) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint4 w = *reinterpret_cast<const uint4 *>(buf + t * D * 2 + ((c ^ (t & (kChunks - 1))) << 4));
                uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                if (ROT) {
                    const uint4 mk = *reinterpret_cast<const uint4 *>(sign_mask + 4 * c);
                    ws[0] ^= mk.x;
                    ws[1] ^= mk.y;
                    ws[2] ^= mk.z;
                    ws[3] ^= mk.w;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[8 * c + 2 * e] = bf16lo(ws[e]);
                    v[8 * c + 2 * e + 1] = bf16hi(ws[e]);
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < D; ++k) v[k] = 0.f;
        }
        if (ROT) {
            // y = v H: butterflies of stride 1 (scalar), then 2, ..., D/2 on
            // packed pairs (each lane rounds as a scalar would)
#pragma unroll
            for (int k = 0; k < D; k += 2) {
                const float p = v[k], q = v[k + 1];
                v[k] = __fadd_rn(p, q);
                v[k + 1] = __fsub_rn(p, q);
            }
#pragma unroll
            for (int h = 2; h < D; h <<= 1)
#pragma unroll
                for (int k = 0; k < D; k += 2)
                    if ((k & h) == 0) {
                        const uint64_t p = f2_pack(v[k], v[k + 1]), q = f2_pack(v[k + h], v[k + h + 1]);
                        f2_unpack(f2_add(p, q), v[k], v[k + 1]);
                        f2_unpack(f2_sub(p, q), v[k + h], v[k + h + 1]);
                    }
        }
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < D; ++k) amax = fmaxf(amax, fabsf(v[k]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((t & 31) == 0) warp_max[t >> 5] = amax;
        __syncthreads();  // also: the previous block's codes have left out_buf
        amax = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
        float r = 1.f;
        if (amax > 0.f) {
            r = __fdiv_rn(448.f, amax);
            if (isinf(r)) r = FLT_MAX;
        }
        if (t == 0) {
            const double den = ROT ? 448.0 * sqrt((double)D) : 448.0;
            scales[(size_t)bh * nblk + b] = amax > 0.f ? __double2float_rn((double)amax / den) : 1.f;
        }
        if (t < rows) {
#pragma unroll
            for (int c = 0; c < kCChunks; ++c) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = 16 * c + 4 * e;
                    const uint32_t lo = pack_e4m3x2(__fmul_rn(v[k], r), __fmul_rn(v[k + 1], r));
                    const uint32_t hi = pack_e4m3x2(__fmul_rn(v[k + 2], r), __fmul_rn(v[k + 3], r));
                    w[e] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4 *>(out_buf + t * D + ((c ^ (t & (kCChunks - 1))) << 4)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        __syncthreads();  // codes staged; every thread is done reading buf and warp_max
        uint4 *dst = reinterpret_cast<uint4 *>(codes + ((size_t)bh * N + r0) * D);
        for (int k = t; k < rows * kCChunks; k += kQRows) {
            const int rr = k / kCChunks, c = k - rr * kCChunks;
            dst[k] = *reinterpret_cast<const uint4 *>(out_buf + rr * D + ((c ^ (rr & (kCChunks - 1))) << 4));
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

}  // namespace

attn_status launch_quantize_fp8(const QuantLaunch &p, cudaStream_t stream) {
    constexpr int D = 128;
    constexpr int kSmem = 2 * kQRows * D * 2 + kQRows * D;  // two bf16 input blocks + one code block
    const int nblk = (p.N + kQRows - 1) / kQRows;
    const long long total = (long long)p.BH * nblk;
    if (total == 0) return ATTN_OK;
    if (total > 0x7fffffffLL) return ATTN_EINVAL;
    static bool attr_set[64] = {false};
    static int sm_count[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(quantize_qk_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(quantize_qk_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
                cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    const long long slots = 2LL * sm_count[dev];  // two resident CTAs per SM
    const int grid = (int)(total < slots ? total : slots);
    const auto *x = static_cast<const __nv_bfloat16 *>(p.x);
    auto *codes = static_cast<uint8_t *>(p.codes);
    if (p.signs)
        quantize_qk_kernel<D, true><<<grid, kQRows, kSmem, stream>>>(x, codes, p.scales, p.signs, p.N, nblk,
                                                                     (int)total);
    else
        quantize_qk_kernel<D, false><<<grid, kQRows, kSmem, stream>>>(x, codes, p.scales, p.signs, p.N, nblk,
                                                                      (int)total);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
