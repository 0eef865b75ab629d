// prefill_sm100.cu -- bf16 dense attention forward (prefill) on sm_100a
// tensor cores: TMA-staged tiles, tcgen05.mma with TMEM accumulators, online
// softmax overlapped with the other query tile's matrix products.
//
// Method (pages): "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
// section 二 核心原理 (Q in row tiles of Br, K/V in column tiles of Bc staged
// in on-chip memory; running max and exp-sum; fused QK^T -> softmax -> PV),
// section 二 FlashAttention-2 改进 (fewer non-matmul operations: one 1/l at
// the end; keep only logsumexp), section 二 FlashAttention-3 改进 (producer
// and consumer warps; softmax hidden under asynchronous block GEMMs).
// "第 2 章核心模块：FlashAttention-2 与 PagedAttention 实现解析" section 2.1
// (incremental normalisation equals one-shot softmax).
//
// What this kernel does on B200 (the pages' versions target A100 / H100):
//   * A CTA owns two 128-row query tiles (Q0, Q1) of one (b, h) and walks the
//     128-key K/V tiles once for both, so each K/V tile is read from L2 once
//     per 256 query rows.
//   * Warp 8 (TMA producer): Q0/Q1 once, then K_j, V_j alternately into a
//     ring of shared-memory slots, 128-byte swizzled, mbarrier completion.
//   * Warp 9 (one elected thread, MMA issuer): S_i = Q_i K_j^T into TMEM
//     (fp32), O_i += P_i V_j into TMEM with P_i taken from TMEM.  Order per
//     key tile: PV0(j), S0(j+1), PV1(j), S1(j+1): while one softmax
//     warpgroup exponentiates, the tensor core works on the other tile.
//   * Warps 0-3 / 4-7 (softmax, one thread per query row): tcgen05.ld the
//     score row, causal / length mask, row max, exp2, bf16 P written back over
//     the scores in TMEM, running sum.  The reference max only moves when the
//     row max grows by more than 2^8 (exact: P and l use the same stale max;
//     the O accumulator is rescaled only then).  Epilogue: O / l, bf16 store,
//     LSE = (m + log2 l) ln 2.
//   TMEM: S0 cols [0,128), S1 [128,256), O0 [256,256+d), O1 [384,384+d).
//   Every mbarrier wait is bounded (1 s) and sets ATTN_DEVERR_TIMEOUT; the
//   kernel then unwinds, waits for its own copies and MMAs, frees TMEM and
//   returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "ptx.cuh"

namespace osp {
namespace {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // keys per tile
constexpr int NQ = 2;          // query tiles per CTA
constexpr int kThreads = 320;  // 2 softmax warpgroups + TMA warp + MMA warp
constexpr int kBoxCols = 64;   // bf16 elements per 128-byte swizzle row
constexpr int kBoxBytes = 128 * 128;  // one box: 128 rows x 128 bytes
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Cfg {
    static constexpr int kBoxes = D / kBoxCols;
    static constexpr int kTileBytes = 128 * D * 2;  // Q, K or V tile
    static constexpr int kStages = D == 128 ? 4 : 8;
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = NQ * kTileBytes;
    static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
    // barriers: q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], done
    static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack
};

struct PrefillArgs {
    __nv_bfloat16 *O;
    float *LSE;
    int32_t *err;
    int N, BH, nblk;
    float scale_log2;
};

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)2 << 61;  // 128-byte swizzle
    return d;
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4)                           // D: fp32
           | (1u << 7)                         // A: bf16
           | (1u << 10)                        // B: bf16
           | ((b_mn_major ? 1u : 0u) << 16)    // B major-ness
           | ((uint32_t)(N >> 3) << 17)        // N / 8
           | ((uint32_t)(M >> 4) << 24);       // M / 16
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, int32_t *err,
                                              volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                if (err) atomicOr(err, ATTN_DEVERR_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
    }
}


// ---------------------------------------------------------------- softmax math

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for a pair of floats on the FMA pipe, keeping the MUFU free for the
// rest.  Range reduction x = n + f with n = round(x) (the 1.5 * 2^23 shift),
// f in [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted to 2^f on [-1/2, 1/2]
// at Chebyshev nodes with relative-error weighting (Lawson iterations towards
// the minimax fit; max relative error 7.5e-5 in fp32, far below the bf16
// rounding of P); 2^n is added into the exponent field.  x is clamped to
// >= -125 so the result stays a normal number (2^-125 ~ 0 next to l >= 1).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    constexpr float c0 = 0x1.fff692p-1f, c1 = 0x1.62f31ap-1f, c2 = 0x1.f0de1ap-3f, c3 = 0x1.c3f75ep-5f;
    float x0, x1;
    f2_unpack(x2, x0, x1);
    x0 = fmaxf(x0, -125.f);
    x1 = fmaxf(x1, -125.f);
    const uint64_t xc = f2_pack(x0, x1);
    const uint64_t t = f2_add(xc, f2_pack(kShift, kShift));           // n in the low mantissa bits
    const uint64_t nr = f2_fma(t, f2_pack(-1.f, -1.f), f2_pack(kShift, kShift));  // -n
    const uint64_t fr = f2_add(xc, nr);                               // f = x - n
    uint64_t r = f2_fma(f2_pack(c3, c3), fr, f2_pack(c2, c2));
    r = f2_fma(r, fr, f2_pack(c1, c1));
    r = f2_fma(r, fr, f2_pack(c0, c0));
    float p0, p1, t0, t1;
    f2_unpack(r, p0, p1);
    f2_unpack(t, t0, t1);
    p0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
    return f2_pack(p0, p1);
}

// Pairs k with (k % 8) >= kPolyFrom take the polynomial; the others MUFU ex2.
constexpr int kPolyFrom = 5;  // 3 of every 8 pairs

// P = 2^(s * scale_log2 - m) for one 128-wide score row held as raw fp32 bits
// in sr, packed to bf16 pairs and stored over the first 64 TMEM columns of
// the row's S region; the fp32 values are summed into acc2 (4 pairs of
// accumulators).  USE_POLY sends 3 of every 8 pairs to the FMA-pipe
// polynomial (only for tiles without masked entries).
template <bool USE_POLY>
__device__ __forceinline__ void exp_pack_store(const uint32_t (&sr)[4][32], uint32_t s_tm, uint64_t scale2,
                                               uint64_t negm2, uint64_t (&acc2)[4]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int c = 2 * h + (e >> 4), k = (e & 15) * 2;
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sr[c][k]), __uint_as_float(sr[c][k + 1])), scale2, negm2);
            uint64_t p2;
            if (USE_POLY && (e & 7) >= kPolyFrom) {
                p2 = exp2_poly2(x2);
            } else {
                float x0, x1;
                f2_unpack(x2, x0, x1);
                p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            acc2[e & 3] = f2_add(acc2[e & 3], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_tm + 32 * h, pk);
    }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, PrefillArgs a) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_full = bars;
    uint64_t *kv_full = bars + 2;
    uint64_t *kv_empty = kv_full + C::kStages;
    uint64_t *s_full = kv_empty + C::kStages;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_full = p_full + 2;
    uint64_t *done_bar = o_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // work unit: longest causal query blocks first
    const int lin = blockIdx.x;
    const int blk = CAUSAL ? (a.nblk - 1 - lin / a.BH) : (lin / a.BH);
    const int bh = lin % a.BH;
    const int n_kv_all = (a.N + BN - 1) / BN;
    int nkv[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int qt = NQ * blk + i;
        nkv[i] = (qt * BM >= a.N) ? 0 : (CAUSAL ? min(qt + 1, n_kv_all) : n_kv_all);
    }
    const int nkv_max = max(nkv[0], nkv[1]);

    if (threadIdx.x == 0) {
        mbar_init(&q_full[0], 1);
        mbar_init(&q_full[1], 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_full[i], 1);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t smem_base = smem_u32(smem);

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            bool ok = true;
            for (int i = 0; i < NQ; ++i) {
                if (nkv[i] == 0) continue;
                uint8_t *dst = smem + C::kQOff + i * C::kTileBytes;
                mbar_arrive_expect_tx(&q_full[i], C::kTileBytes);
                for (int b = 0; b < C::kBoxes; ++b)
                    tma_load_3d(dst + b * kBoxBytes, &tmQ, &q_full[i], b * kBoxCols, (NQ * blk + i) * BM, bh);
            }
            const int n_loads = 2 * nkv_max;
            int u = 0;
            for (; u < n_loads && ok; ++u) {
                const int slot = u % C::kStages;
                if (u >= C::kStages) ok = wait_or_abort(&kv_empty[slot], ((u / C::kStages) - 1) & 1, a.err, abort_flag);
                if (!ok) break;
                const int j = u >> 1;
                const CUtensorMap *tm = (u & 1) ? &tmV : &tmK;
                uint8_t *dst = smem + C::kRingOff + slot * C::kTileBytes;
                mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
                for (int b = 0; b < C::kBoxes; ++b)
                    tma_load_3d(dst + b * kBoxBytes, tm, &kv_full[slot], b * kBoxCols, j * BN, bh);
            }
            // copies still in flight must land before the CTA can exit: wait
            // (bounded) for the newest phase of every slot that was loaded
            for (int v = max(0, u - C::kStages); v < u; ++v)
                mbar_wait(&kv_full[v % C::kStages], (v / C::kStages) & 1, nullptr);
            for (int i = 0; i < NQ; ++i)
                if (nkv[i] > 0) mbar_wait(&q_full[i], 0, nullptr);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
            const uint32_t q_addr = smem_base + C::kQOff;
            const uint32_t ring_addr = smem_base + C::kRingOff;
            bool ok = true;
            auto slot_addr = [&](int u) { return ring_addr + (u % C::kStages) * C::kTileBytes; };
            auto wait_kv = [&](int u) {
                return wait_or_abort(&kv_full[u % C::kStages], (u / C::kStages) & 1, a.err, abort_flag);
            };
            auto issue_s = [&](int i, int u) {
                const uint32_t qa = q_addr + i * C::kTileBytes, ka = slot_addr(u);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * kBoxBytes + (ks % 4) * 32;
                    mma_ss(tmem + i * BN, desc_sw128(qa + off, 16, 1024), desc_sw128(ka + off, 16, 1024), idesc_qk,
                           ks > 0);
                }
                mma_commit(&s_full[i]);
            };
            auto issue_pv = [&](int i, int u, int j) {
                const uint32_t va = slot_addr(u);
#pragma unroll
                for (int ks = 0; ks < BN / 16; ++ks) {
                    mma_ts(tmem + 2 * BN + i * 128, tmem + i * BN + ks * 8,
                           desc_sw128(va + ks * 16 * 128, kBoxBytes, 1024), idesc_pv, (j > 0 || ks > 0));
                }
                mma_commit(&o_full[i]);
            };
            for (int i = 0; i < NQ && ok; ++i)
                if (nkv[i] > 0) ok = wait_or_abort(&q_full[i], 0, a.err, abort_flag);
            if (ok) ok = wait_kv(0);
            if (ok) {
                tc_fence_after();
                for (int i = 0; i < NQ; ++i)
                    if (nkv[i] > 0) issue_s(i, 0);
                mma_commit(&kv_empty[0]);
            }
            for (int j = 0; j < nkv_max && ok; ++j) {
                const int uV = 2 * j + 1, uK = 2 * j + 2;
                ok = wait_kv(uV);
                if (!ok) break;
                bool k_ready = false;
                for (int i = 0; i < NQ && ok; ++i) {
                    if (j >= nkv[i]) continue;
                    ok = wait_or_abort(&p_full[i], j & 1, a.err, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(i, uV, j);
                    if (j + 1 < nkv[i]) {
                        if (!k_ready) {
                            ok = wait_kv(uK);
                            if (!ok) break;
                            tc_fence_after();
                            k_ready = true;
                        }
                        issue_s(i, uK);
                    }
                }
                if (!ok) break;
                mma_commit(&kv_empty[uV % C::kStages]);
                if (j + 1 < nkv_max) {
                    if (!k_ready) {
                        ok = wait_kv(uK);
                        if (!ok) break;
                    }
                    mma_commit(&kv_empty[uK % C::kStages]);
                }
            }
            // every MMA issued by this thread has completed before TMEM is freed
            mma_commit(done_bar);
            mbar_wait(done_bar, 0, nullptr);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int i = warp >> 2;                 // query tile of this warpgroup
        const int quarter = warp & 3;            // TMEM lane quarter
        const int r = quarter * 32 + lane;       // row inside the tile
        const int qt = NQ * blk + i;
        const int row = qt * BM + r;             // query row in the sequence
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_tm = tmem + lane_off + i * BN;
        const uint32_t o_tm = tmem + lane_off + 2 * BN + i * 128;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        const int my_nkv = i ? nkv[1] : nkv[0];
        for (int j = 0; j < my_nkv; ++j) {
            ok = wait_or_abort(&s_full[i], j & 1, a.err, abort_flag);
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + 32 * c, sr[c]);
            tmem_wait_ld();
            // visible keys: col <= lim; only the causal diagonal tile and the
            // sequence's last tile need masking
            const bool masked = (CAUSAL && j == qt) || ((j + 1) * BN > a.N);
            if (masked) {
                int lim = BN - 1;
                if (CAUSAL && j == qt) lim = r;
                lim = min(lim, a.N - 1 - j * BN);
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * c + e > lim) sr[c][e] = __float_as_uint(-INFINITY);
            }
            float mxa[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mxa[k] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    const int k = (e >> 3) + 4 * (c & 1);
                    mxa[k] = max3(mxa[k], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
                    mxa[k] = max3(mxa[k], __uint_as_float(sr[c][e + 2]), __uint_as_float(sr[c][e + 3]));
                    mxa[k] = max3(mxa[k], __uint_as_float(sr[c][e + 4]), __uint_as_float(sr[c][e + 5]));
                    mxa[k] = max3(mxa[k], __uint_as_float(sr[c][e + 6]), __uint_as_float(sr[c][e + 7]));
                }
            const float mx = max3(max3(mxa[0], mxa[1], mxa[2]), max3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
            const float mx2 = mx * a.scale_log2;
            float m_ref = m;
            if (mx2 > m + kRescaleThreshold) m_ref = mx2;
            if (m_ref == -INFINITY) m_ref = 0.f;  // row with nothing visible yet
            const float alpha = ex2_approx(m - m_ref);
            const uint64_t scale2 = f2_pack(a.scale_log2, a.scale_log2);
            const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
            uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
            if (masked)
                exp_pack_store<false>(sr, s_tm, scale2, negm2, acc2);
            else
                exp_pack_store<true>(sr, s_tm, scale2, negm2, acc2);
            float psum;
            {
                const uint64_t t2 = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
                float u0, u1;
                f2_unpack(t2, u0, u1);
                psum = u0 + u1;
            }
            l = l * alpha + psum;
            const bool need = (m_ref != m) && j > 0;
            if (__any_sync(0xffffffffu, need)) {
                // PV(j-1) has completed: S(j) was issued after it and has landed
                ok = wait_or_abort(&o_full[i], (j - 1) & 1, a.err, abort_flag);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t orr[32];
                    tmem_ld32(o_tm + 32 * c, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                    tmem_st32(o_tm + 32 * c, orr);
                }
            }
            m = m_ref;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[i]);
        }
        if (ok && my_nkv > 0) {
            ok = wait_or_abort(&o_full[i], (my_nkv - 1) & 1, a.err, abort_flag);
            if (ok) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const bool live = row < a.N;
                __nv_bfloat16 *orow = a.O + ((size_t)bh * a.N + (live ? row : 0)) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t orr[32];
                    tmem_ld32(o_tm + 32 * c, orr);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
                    if (live) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
                if (live)
                    a.LSE[(size_t)bh * a.N + row] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B*H, N, d] bf16 viewed as a 3-D tensor map, box 64 x 128 x 1, 128B swizzle.
bool make_map(CUtensorMap *m, const void *base, int N, int d, int BH) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {kBoxCols, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool CAUSAL>
attn_status launch_t(const DenseLaunch &p, cudaStream_t stream) {
    using C = Cfg<D>;
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(prefill_bf16_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    CUtensorMap tq, tk, tv;
    const int BH = p.B * p.H;
    if (!make_map(&tq, p.Q, p.N, D, BH) || !make_map(&tk, p.K, p.N, D, BH) || !make_map(&tv, p.V, p.N, D, BH))
        return ATTN_ECUDA;
    PrefillArgs a;
    a.O = static_cast<__nv_bfloat16 *>(p.O);
    a.LSE = p.LSE;
    a.err = p.err_flag;
    a.N = p.N;
    a.BH = BH;
    a.nblk = (p.N + NQ * BM - 1) / (NQ * BM);
    a.scale_log2 = p.scale * 1.4426950408889634f;
    const long long grid = (long long)a.nblk * BH;
    prefill_bf16_kernel<D, CAUSAL><<<(unsigned)grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace

attn_status launch_prefill_bf16(const DenseLaunch &p, cudaStream_t stream) {
    if (p.d == 128) return p.causal ? launch_t<128, true>(p, stream) : launch_t<128, false>(p, stream);
    return p.causal ? launch_t<64, true>(p, stream) : launch_t<64, false>(p, stream);
}

}  // namespace osp
