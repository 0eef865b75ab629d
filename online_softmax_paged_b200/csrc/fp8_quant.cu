// fp8_quant.cu -- block quantisation of Q or K to e4m3, with optional
// incoherent processing, for the FP8 prefill.
//
// Method (pages): "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
// §二 "FlashAttention-3改进": the forward pass runs its GEMMs on FP8 tensor
// cores, and block quantisation plus incoherent processing limit the accuracy
// lost in the conversion.  Here the QK^T product is the FP8 one.
//
// One CTA per (head, 128-row block), one thread per row.  Per block:
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

template <int D, bool ROT>
__global__ void __launch_bounds__(kQRows) quantize_qk_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             uint8_t *__restrict__ codes, float *__restrict__ scales,
                                                             const int8_t *__restrict__ signs, int N, int nblk) {
    constexpr int kChunks = D / 8;  // 16-byte chunks of a bf16 row
    __shared__ __align__(16) uint8_t buf[kQRows * D * 2];
    __shared__ float warp_max[kQRows / 32];
    __shared__ __align__(16) uint32_t sign_mask[D / 2];  // per bf16x2 word: the sign bits to flip
    const int t = threadIdx.x;
    const int bh = blockIdx.x / nblk, b = blockIdx.x - bh * nblk;
    const int r0 = b * kQRows;
    const int rows = min(kQRows, N - r0);
    const size_t base = ((size_t)bh * N + r0) * D;

    // coalesced load of the block (rows * D bf16, contiguous)
    if (ROT && t < D / 2)
        sign_mask[t] = (__ldg(signs + 2 * t) < 0 ? 0x8000u : 0u) | (__ldg(signs + 2 * t + 1) < 0 ? 0x80000000u : 0u);
    const uint4 *src = reinterpret_cast<const uint4 *>(x + base);
    for (int k = t; k < rows * kChunks; k += kQRows) {
        const int r = k / kChunks, c = k - r * kChunks;
        *reinterpret_cast<uint4 *>(buf + r * D * 2 + ((c ^ (r & (kChunks - 1))) << 4)) = __ldg(src + k);
    }
    __syncthreads();

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
    __syncthreads();  // every thread is done reading buf as well
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
    // codes of row t -> shared (swizzled 16-byte chunks), then coalesced out
    constexpr int kCChunks = D / 16;  // 16-byte chunks of a code row
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
            *reinterpret_cast<uint4 *>(buf + t * D + ((c ^ (t & (kCChunks - 1))) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    __syncthreads();
    uint4 *dst = reinterpret_cast<uint4 *>(codes + base);
    for (int k = t; k < rows * kCChunks; k += kQRows) {
        const int rr = k / kCChunks, c = k - rr * kCChunks;
        dst[k] = *reinterpret_cast<const uint4 *>(buf + rr * D + ((c ^ (rr & (kCChunks - 1))) << 4));
    }
}

}  // namespace

attn_status launch_quantize_fp8(const QuantLaunch &p, cudaStream_t stream) {
    const int nblk = (p.N + kQRows - 1) / kQRows;
    const long long grid = (long long)p.BH * nblk;
    if (grid == 0) return ATTN_OK;
    if (grid > 0x7fffffffLL) return ATTN_EINVAL;
    const auto *x = static_cast<const __nv_bfloat16 *>(p.x);
    auto *codes = static_cast<uint8_t *>(p.codes);
    if (p.signs)
        quantize_qk_kernel<128, true><<<(unsigned)grid, kQRows, 0, stream>>>(x, codes, p.scales, p.signs, p.N, nblk);
    else
        quantize_qk_kernel<128, false><<<(unsigned)grid, kQRows, 0, stream>>>(x, codes, p.scales, p.signs, p.N, nblk);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
