// dense_f32.cu -- fp32 dense attention forward on CUDA cores (FFMA), causal
// or not.  fp32 is kept exact to fp32 rounding: no TF32 tensor-core path,
// whose 10-bit mantissa could not meet a 1e-4 bound.
//
// Method: "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
// section 二 核心原理 (Q split into row tiles, K/V into column tiles staged in
// on-chip memory, running max and exp-sum per row), "第 2 章核心模块：
// FlashAttention-2 与 PagedAttention 实现解析" section 2.1 (incremental
// normalisation; FA-2's single 1/l at the end).
//
// Layout: a CTA owns 32 query rows of one (b, h); four threads share a row,
// thread q of the quad holding float4 chunks q, q+4, q+8, ... of the row so a
// quad reads 64 contiguous bytes of a shared K/V row (broadcast across rows,
// no bank conflicts).  K/V tiles of 32 keys are staged in shared memory.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "launch.h"
#include "ptx.cuh"

namespace osp {
namespace {

constexpr int kRows = 32;
constexpr int kKeys = 32;

template <int D>
__global__ void __launch_bounds__(128) dense_f32_kernel(const float *__restrict__ Q, const float *__restrict__ K,
                                                        const float *__restrict__ V, float *__restrict__ O,
                                                        float *__restrict__ LSE, int N, int causal,
                                                        float scale_log2) {
    constexpr int C4 = D / 4;        // float4 chunks per row
    constexpr int MY = C4 / 4;       // chunks per thread
    __shared__ float4 Ks[kKeys][C4];
    __shared__ float4 Vs[kKeys][C4];

    const int tid = threadIdx.x;
    const int r_local = tid >> 2, qd = tid & 3;
    const int row0 = blockIdx.x * kRows;
    const int row = row0 + r_local;
    const size_t bh = (size_t)blockIdx.z * gridDim.y + blockIdx.y;
    const float4 *Qg = reinterpret_cast<const float4 *>(Q + bh * N * D);
    const float4 *Kg = reinterpret_cast<const float4 *>(K + bh * N * D);
    const float4 *Vg = reinterpret_cast<const float4 *>(V + bh * N * D);

    float4 q[MY], o[MY];
#pragma unroll
    for (int i = 0; i < MY; ++i) {
        q[i] = row < N ? Qg[(size_t)row * C4 + 4 * i + qd] : make_float4(0.f, 0.f, 0.f, 0.f);
        q[i].x *= scale_log2; q[i].y *= scale_log2; q[i].z *= scale_log2; q[i].w *= scale_log2;
        o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float m = -INFINITY, l = 0.f;

    const int key_end = causal ? min(N, row0 + kRows) : N;
    for (int j0 = 0; j0 < key_end; j0 += kKeys) {
        __syncthreads();
        for (int e = tid; e < kKeys * C4; e += 128) {
            const int j = e / C4, c = e % C4;
            const bool in = j0 + j < N;
            Ks[j][c] = in ? Kg[(size_t)(j0 + j) * C4 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
            Vs[j][c] = in ? Vg[(size_t)(j0 + j) * C4 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        float s[kKeys];
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < kKeys; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < MY; ++i) {
                const float4 k = Ks[j][4 * i + qd];
                acc = fmaf(q[i].x, k.x, acc);
                acc = fmaf(q[i].y, k.y, acc);
                acc = fmaf(q[i].z, k.z, acc);
                acc = fmaf(q[i].w, k.w, acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            const int key = j0 + j;
            const bool vis = key < N && (!causal || key <= row);
            s[j] = vis ? acc : -INFINITY;
            mt = fmaxf(mt, s[j]);
        }
        const float m_new = fmaxf(m, mt);
        if (m_new == -INFINITY) continue;  // nothing visible yet (rows past N / causal)
        const float alpha = ex2_approx(m - m_new);
        float psum = 0.f;
#pragma unroll
        for (int j = 0; j < kKeys; ++j) {
            s[j] = ex2_approx(s[j] - m_new);
            psum += s[j];
        }
        l = l * alpha + psum;
#pragma unroll
        for (int i = 0; i < MY; ++i) {
            o[i].x *= alpha; o[i].y *= alpha; o[i].z *= alpha; o[i].w *= alpha;
        }
#pragma unroll
        for (int j = 0; j < kKeys; ++j) {
            const float p = s[j];
#pragma unroll
            for (int i = 0; i < MY; ++i) {
                const float4 v = Vs[j][4 * i + qd];
                o[i].x = fmaf(p, v.x, o[i].x);
                o[i].y = fmaf(p, v.y, o[i].y);
                o[i].z = fmaf(p, v.z, o[i].z);
                o[i].w = fmaf(p, v.w, o[i].w);
            }
        }
        m = m_new;
    }
    if (row < N) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float4 *Og = reinterpret_cast<float4 *>(O + bh * N * D);
#pragma unroll
        for (int i = 0; i < MY; ++i)
            Og[(size_t)row * C4 + 4 * i + qd] = make_float4(o[i].x * inv, o[i].y * inv, o[i].z * inv, o[i].w * inv);
        if (qd == 0)
            LSE[bh * N + row] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
}

}  // namespace

attn_status launch_dense_f32(const DenseLaunch &p, cudaStream_t stream) {
    dim3 grid((p.N + kRows - 1) / kRows, p.H, p.B);
    const float sl2 = p.scale * 1.4426950408889634f;
    const float *Q = static_cast<const float *>(p.Q);
    const float *K = static_cast<const float *>(p.K);
    const float *V = static_cast<const float *>(p.V);
    float *O = static_cast<float *>(p.O);
    if (p.d == 64)
        dense_f32_kernel<64><<<grid, 128, 0, stream>>>(Q, K, V, O, p.LSE, p.N, p.causal, sl2);
    else
        dense_f32_kernel<128><<<grid, 128, 0, stream>>>(Q, K, V, O, p.LSE, p.N, p.causal, sl2);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
