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
//     per 256 query rows.  In a bf16 causal unit Q0 is the later 128 rows
//     (one key tile more), so the tile the MMA warp serves first at each key
//     step is also the one that ends the unit.
//   * Warp 8 (TMA producer): Q0/Q1 once, then K_j, V_j alternately into a
//     ring of shared-memory slots, 128-byte swizzled, mbarrier completion.
//   * Warp 9 (one elected thread, MMA issuer): S_i = Q_i K_j^T into TMEM
//     (fp32), O_i += P_i V_j into TMEM with P_i taken from TMEM.  Order per
//     key tile: PV0(j), S0(j+1), PV1(j), S1(j+1): while one softmax
//     warpgroup exponentiates, the tensor core works on the other tile.
//   * Warps 0-3 / 4-7 (softmax, one thread per query row): tcgen05.ld the
//     score row (two 64-column loads), causal / length mask, row max, exp2
//     (2 of every 8 pairs by an FMA-pipe polynomial, the rest on the
//     special-function unit), bf16 P written back over the scores in TMEM,
//     running sum.  The reference max only moves when the
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
#include "softmax_math.cuh"

namespace osp {
namespace {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // keys per tile
constexpr int NQ = 2;          // query tiles per CTA
constexpr int kThreads = 384;  // 2 softmax warpgroups + a producer warpgroup (TMA warp, MMA warp, 2 idle)
// Register split (setmaxnreg, executed inside each role's branch): launched
// at 168 per thread (384 x 168 = 64512); the producer warpgroup drops to 64
// and each softmax warpgroup rises to 208: 128 x 64 + 256 x 208 = 61440.
constexpr int kProducerRegs = 64;
constexpr int kSoftmaxRegs = 208;
static_assert(128 * kProducerRegs + 2 * 128 * kSoftmaxRegs <= kThreads * 168, "register split over budget");
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
    // one O tile (D / 64 boxes of 64 columns) staged for the TMA store, shared
    // by the two query tiles in unit order
    static constexpr int kStageOff = kRingOff + kStages * kTileBytes;
    static constexpr int kBarOff = kStageOff + kBoxes * kBoxBytes;
    // barriers: q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], done,
    // stg_full[2], stg_free[2]
    static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 1 + 2 + 2;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct PrefillArgs {
    __nv_bfloat16 *O;
    float *LSE;
    int32_t *err;
    int N, BH, nblk;
    float scale_log2;
    // paged mode: query tokens of sequence s are rows cu_q[s] .. cu_q[s+1]-1 of
    // q / O / LSE, at key positions seq_lens[s] - n_s .. seq_lens[s] - 1
    const int32_t *cu_q, *seq_lens, *block_table;
    int S, Hq, Hkv, max_blocks, num_blocks, block_size, nqb, total_q;
    // FP8 mode: e4m3 Q and K with one dequantisation scale per 128-row block
    // ([B*H, nsblk] each); V stays bf16
    const float *q_scale, *k_scale;
    int nsblk;
};

// What every role needs to know about a work unit (256 query rows of one
// head).  Dense: rows qrow0 .. of head `head` ((b, h) flattened), keys 0 .. N-1.
// Paged: rows qrow0 .. of sequence s's new tokens, query head `head`,
// key/value head kv_head, keys 0 .. L-1, row r at key position pos0 + r.
struct UnitInfo {
    int head, kv_head, s, qrow0, nq, pos0, L, qtok0;
    int row0[2];  // first row of query tile 0 / 1 (qrow0 + 128 and qrow0 when causal, see get_unit)
    int n0, n1;   // key tiles of query tile 0 / 1 (0: the tile has no rows)
    int bad;      // paged: device error bits of an inconsistent sequence (0: fine)
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

// kind::f8f6f4 instruction descriptor: e4m3 A and B, both K-major, fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4)                           // D: fp32
           | (0u << 7)                         // A: e4m3
           | (0u << 10)                        // B: e4m3
           | ((uint32_t)(N >> 3) << 17)        // N / 8
           | ((uint32_t)(M >> 4) << 24);       // M / 16
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


// 32 lanes x 64 consecutive 32-bit columns in one load: columns 0-31 of the
// group to lo, 32-63 to hi (thread t gets lane base + t).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&lo)[32], uint32_t (&hi)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(lo[0]), "=r"(lo[1]), "=r"(lo[2]), "=r"(lo[3]), "=r"(lo[4]), "=r"(lo[5]), "=r"(lo[6]), "=r"(lo[7]),
          "=r"(lo[8]), "=r"(lo[9]), "=r"(lo[10]), "=r"(lo[11]), "=r"(lo[12]), "=r"(lo[13]), "=r"(lo[14]), "=r"(lo[15]),
          "=r"(lo[16]), "=r"(lo[17]), "=r"(lo[18]), "=r"(lo[19]), "=r"(lo[20]), "=r"(lo[21]), "=r"(lo[22]), "=r"(lo[23]),
          "=r"(lo[24]), "=r"(lo[25]), "=r"(lo[26]), "=r"(lo[27]), "=r"(lo[28]), "=r"(lo[29]), "=r"(lo[30]), "=r"(lo[31]),
          "=r"(hi[0]), "=r"(hi[1]), "=r"(hi[2]), "=r"(hi[3]), "=r"(hi[4]), "=r"(hi[5]), "=r"(hi[6]), "=r"(hi[7]),
          "=r"(hi[8]), "=r"(hi[9]), "=r"(hi[10]), "=r"(hi[11]), "=r"(hi[12]), "=r"(hi[13]), "=r"(hi[14]), "=r"(hi[15]),
          "=r"(hi[16]), "=r"(hi[17]), "=r"(hi[18]), "=r"(hi[19]), "=r"(hi[20]), "=r"(hi[21]), "=r"(hi[22]), "=r"(hi[23]),
          "=r"(hi[24]), "=r"(hi[25]), "=r"(hi[26]), "=r"(hi[27]), "=r"(hi[28]), "=r"(hi[29]), "=r"(hi[30]), "=r"(hi[31])
        : "r"(taddr));
}

// Pairs k with (k % 8) >= kPolyFrom take the polynomial; the others MUFU ex2.
constexpr int kPolyFrom = 6;  // 2 of every 8 pairs (re-measured against 1 and 3 of 8)

// P = 2^(s * scale_log2 - m) for one 128-wide score row held as raw fp32 bits
// in sr, packed to bf16 pairs and stored over the first 64 TMEM columns of
// the row's S region; the fp32 values are summed into acc2 (4 pairs of
// accumulators).  2 of every 8 pairs go to the FMA-pipe polynomial, masked
// tiles included: a masked score (-inf) comes out of its clamp as 2^-125
// instead of 0, which adds nothing visible to a running sum l >= 1 or to O
// (the V rows under masked keys are finite: real keys, zero-filled rows
// past N, and the zeroed dead rows of a paged sequence's last tile).
__device__ __forceinline__ void exp_pack_store(const uint32_t (&sr)[4][32], uint32_t s_tm, uint64_t scale2,
                                               uint64_t negm2, uint64_t (&acc2)[4]) {
    // one 32-score chunk at a time: its 16 packed words are stored before the
    // next chunk is exponentiated, so the chunk's registers are free again
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), scale2, negm2);
            uint64_t p2;
            if (((e + 16 * c) & 7) >= kPolyFrom) {
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
        tmem_st16(s_tm + 16 * c, pk);
    }
}

// Work unit u (a 256-row query block of one (b, h)) -> its block index and
// (b, h); causal units are numbered longest first.
__device__ __forceinline__ void unit_coords(const PrefillArgs &a, bool causal, int u, int &blk, int &bh) {
    blk = causal ? (a.nblk - 1 - u / a.BH) : (u / a.BH);
    bh = u % a.BH;
}

// The r-th unit of CTA c in snake order over rows of gridDim.x units
// (row-major rows, every other row reversed), or -1 past the end.
__device__ __forceinline__ int snake_unit(int r, int c, int G, int n_units) {
    const int u = r * G + ((r & 1) ? (G - 1 - c) : c);
    return u < n_units ? u : -1;
}

// Unit u of the kernel's unit space -> UnitInfo.  Dense units are numbered
// longest first when causal; paged units as (sequence, query block, head)
// with later query blocks (more keys) first.  A paged unit past its
// sequence's new tokens, or of an inconsistent sequence, gets n0 = n1 = 0;
// the latter also gets `bad` (cu_q outside [0, total_q] or decreasing:
// ATTN_DEVERR_INDEX; more new tokens than cached keys, or more keys than the
// table holds: ATTN_DEVERR_SEQ_LEN).
template <bool PAGED>
__device__ __forceinline__ void get_unit(const PrefillArgs &a, bool causal, int u, UnitInfo &x, bool later_first) {
    x.bad = 0;
    if (!PAGED) {
        int blk;
        unit_coords(a, causal, u, blk, x.head);
        x.kv_head = x.head;
        x.s = 0;
        x.qrow0 = NQ * BM * blk;
        x.nq = x.L = a.N;
        x.pos0 = 0;
        x.qtok0 = 0;
    } else {
        // sequence-major, so that the CTAs at work at any time share one or
        // two sequences' K/V in L2; within a sequence the later (longer)
        // query blocks first, then the query heads (a key/value head's group
        // adjacent)
        const int per_seq = a.nqb * a.Hq;
        x.s = u / per_seq;
        const int rem = u - x.s * per_seq;
        const int qb = a.nqb - 1 - rem / a.Hq;
        x.head = rem - (rem / a.Hq) * a.Hq;
        x.kv_head = x.head / (a.Hq / a.Hkv);
        x.qtok0 = a.cu_q[x.s];
        x.nq = a.cu_q[x.s + 1] - x.qtok0;
        x.L = a.seq_lens[x.s];
        x.pos0 = x.L - x.nq;
        x.qrow0 = NQ * BM * qb;
        if (x.qtok0 < 0 || x.nq < 0 || x.qtok0 + x.nq > a.total_q) x.bad = ATTN_DEVERR_INDEX;
        else if (x.pos0 < 0 || (long long)x.L > (long long)a.max_blocks * a.block_size) x.bad = ATTN_DEVERR_SEQ_LEN;
    }
    const int n_kv_all = (x.L + BN - 1) / BN;
    // later_first (bf16 causal units): tile 0 takes the unit's later 128
    // rows, which see one key tile more.  The MMA warp works through a unit's
    // key tiles in order, tile 0 before tile 1 at each step, so the tile with
    // the extra (diagonal) step is the one it serves first: once that step's
    // P.V is issued the next unit's first QK^T products follow at once,
    // instead of tile 0 waiting behind tile 1's extra softmax (+2.5-3 % at
    // 2k, measured; the FP8 mode, whose QK^T is twice as fast, measured it
    // neutral and keeps the plain order).
    x.row0[0] = x.qrow0 + (later_first ? BM : 0);
    x.row0[1] = x.qrow0 + (later_first ? 0 : BM);
    int n[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int r0 = x.row0[i];
        n[i] = (x.bad || r0 >= x.nq) ? 0
               : (causal ? min((x.pos0 + r0 + BM - 1) / BN + 1, n_kv_all) : n_kv_all);
    }
    x.n0 = n[0];
    x.n1 = n[1];
}

template <int D, bool CAUSAL, bool PAGED, bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                        PrefillArgs a) {
    using C = Cfg<D>;
    static_assert(!F8 || (D == 128 && !PAGED), "FP8 QK^T: dense, d = 128");
    constexpr bool kLaterFirst = CAUSAL && !F8;  // see get_unit
    // Q and K tiles: bf16 in 64-column boxes, or e4m3 in one 128-byte-wide box
    constexpr int kQKBytes = F8 ? BM * D : C::kTileBytes;
    constexpr int kQKBoxes = F8 ? 1 : C::kBoxes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *q_full = bars;
    uint64_t *q_empty = q_full + 2;
    uint64_t *kv_full = q_empty + 2;
    uint64_t *kv_empty = kv_full + C::kStages;
    uint64_t *s_full = kv_empty + C::kStages;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_full = p_full + 2;
    uint64_t *done_bar = o_full + 2;
    uint64_t *stg_full = done_bar + 1;  // [tile] the tile's 128 rows are in the staging buffer
    uint64_t *stg_free = stg_full + 2;  // [0] the last TMA store has read the staging buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int n_units = PAGED ? a.nqb * a.S * a.Hq : a.nblk * a.BH;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_full[i], 1);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(done_bar, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&stg_full[i], 128);
            mbar_init(&stg_free[i], 1);
        }
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
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        {
            if (elect_one()) {
                prefetch_tmap(&tmQ);
                prefetch_tmap(&tmK);
                prefetch_tmap(&tmV);
            }
            bool ok = true;
            uint32_t ukv = 0;         // K/V tiles loaded so far (ring position)
            uint32_t qc[2] = {0, 0};  // Q tiles loaded so far, per query tile
            // dense L2 policy: a Q tile is read by one unit only (streamed),
            // while a head's K/V tiles are re-read by every unit of the head
            // (kept): without the hints the Q and O streams pushed K/V out of
            // L2 and K/V was read from DRAM about 1.6 times over at 2k
            const uint64_t pol_stream = l2_policy_evict_first(), pol_keep = l2_policy_evict_last();
            for (int r = 0; ok; ++r) {
                const int u = snake_unit(r, c, G, n_units);
                if (u < 0) break;
                UnitInfo x;
                get_unit<PAGED>(a, CAUSAL, u, x, kLaterFirst);
                const int n0 = x.n0, n1 = x.n1;
                if (PAGED && x.bad && x.qrow0 == 0 && x.head == 0 && elect_one() && a.err)
                    atomicOr(a.err, x.bad);
                auto load_q = [&](int i) {
                    if ((i ? n1 : n0) == 0) return;
                    // the previous unit's QK^T products of this tile are done
                    if (qc[i] > 0) ok = wait_or_abort(&q_empty[i], (qc[i] - 1) & 1, a.err, abort_flag);
                    if (!ok) return;
                    uint8_t *dst = smem + C::kQOff + i * C::kTileBytes;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&q_full[i], kQKBytes);
                        for (int b = 0; b < kQKBoxes; ++b) {
                            if (PAGED)  // rows past the sequence's tokens are loaded but never stored
                                tma_load_2d(dst + b * kBoxBytes, &tmQ, &q_full[i], x.head * D + b * kBoxCols,
                                            x.qtok0 + x.row0[i]);
                            else
                                tma_load_3d_hint(dst + b * kBoxBytes, &tmQ, &q_full[i], b * kBoxCols,
                                                 x.row0[i], x.head, pol_stream);
                        }
                    }
                    __syncwarp();
                    ++qc[i];
                };
                // dense: order Q0, K0, Q1, V0, K1, ...: Q1 is released last (by
                // the previous unit's final QK^T) and must not hold back K0,
                // which tile 0's first QK^T of this unit needs early.  Paged K
                // tiles take one table read and 128 / block_size copies each;
                // there Q0, Q1, K0 measured faster.
                load_q(0);
                if (PAGED) load_q(1);
                const int n_loads = 2 * max(n0, n1);
                for (int v = 0; v < n_loads && ok; ++v, ++ukv) {
                    if (!PAGED && v == 1) {
                        load_q(1);
                        if (!ok) break;
                    }
                    const int slot = ukv % C::kStages;
                    if (ukv >= (uint32_t)C::kStages)
                        ok = wait_or_abort(&kv_empty[slot], ((ukv / C::kStages) - 1) & 1, a.err, abort_flag);
                    if (!ok) break;
                    const CUtensorMap *tm = (v & 1) ? &tmV : &tmK;
                    uint8_t *dst = smem + C::kRingOff + slot * C::kTileBytes;
                    if (!PAGED) {
                        const bool qk = F8 && !(v & 1);  // an e4m3 K tile
                        if (elect_one()) {
                            mbar_arrive_expect_tx(&kv_full[slot], qk ? kQKBytes : C::kTileBytes);
                            for (int b = 0; b < (qk ? kQKBoxes : C::kBoxes); ++b)
                                tma_load_3d_hint(dst + b * kBoxBytes, tm, &kv_full[slot], b * kBoxCols,
                                                 (v >> 1) * BN, x.head, pol_keep);
                        }
                    } else {
                        // one box per cache block: lane k loads block k of the tile.
                        // Blocks past the sequence load its block 0 instead (finite
                        // data under masked keys); ids outside the pool use block 0
                        // and are reported.
                        const int per = BN / a.block_size;
                        const int lb0 = (v >> 1) * per;
                        const int nblk_seq = (x.L + a.block_size - 1) / a.block_size;
                        int phys = 0;
                        if (lane < per) {
                            const int32_t *row = a.block_table + (size_t)x.s * a.max_blocks;
                            phys = row[lb0 + lane < nblk_seq ? lb0 + lane : 0];
                            if (phys < 0 || phys >= a.num_blocks) {
                                if (a.err) atomicOr(a.err, ATTN_DEVERR_BLOCK_TABLE);
                                phys = 0;
                            }
                        }
                        if (elect_one()) mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
                        __syncwarp();
                        if (lane < per) {
                            const int y = (phys * a.Hkv + x.kv_head) * a.block_size;
                            for (int b = 0; b < C::kBoxes; ++b)
                                tma_load_2d(dst + b * kBoxBytes + lane * a.block_size * 128, tm, &kv_full[slot],
                                            b * kBoxCols, y);
                        }
                        __syncwarp();
                    }
                }
            }
            // copies still in flight must land before the CTA can exit: wait
            // (bounded) for the newest phase of every slot and Q buffer loaded
            const uint32_t first = ukv > (uint32_t)C::kStages ? ukv - C::kStages : 0u;
            for (uint32_t v = first; v < ukv; ++v)
                mbar_wait(&kv_full[v % C::kStages], (v / C::kStages) & 1, nullptr);
            if (qc[0] > 0) mbar_wait(&q_full[0], (qc[0] - 1) & 1, nullptr);
            if (qc[1] > 0) mbar_wait(&q_full[1], (qc[1] - 1) & 1, nullptr);
            __syncwarp();
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
        {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
            constexpr uint32_t idesc_qk8 = idesc_e4m3_f32(BM, BN);
            // base descriptors; per-slot and per-k-step offsets are added to the
            // start-address field (16-byte units, no carry: smem < 256 KiB)
            const uint64_t dq0 = desc_sw128(smem_base + C::kQOff, 16, 1024);
            const uint64_t dq1 = desc_sw128(smem_base + C::kQOff + C::kTileBytes, 16, 1024);
            const uint64_t dk = desc_sw128(smem_base + C::kRingOff, 16, 1024);
            const uint64_t dv = desc_sw128(smem_base + C::kRingOff, kBoxBytes, 1024);
            const uint32_t tm_s0 = tmem, tm_s1 = tmem + BN, tm_o0 = tmem + 2 * BN, tm_o1 = tmem + 2 * BN + 128;
            bool ok = true;
            uint32_t ukv = 0;              // K/V ring position (same order as the producer)
            uint32_t qc0 = 0, qc1 = 0;     // Q tiles consumed, per query tile
            uint32_t it0 = 0, it1 = 0;     // key-tile iterations done, per query tile
            auto slot_off = [&](uint32_t u) -> uint64_t { return (uint64_t)(((u % C::kStages) * C::kTileBytes) >> 4); };
            auto wait_kv = [&](uint32_t u) {
                return wait_or_abort(&kv_full[u % C::kStages], (u / C::kStages) & 1, a.err, abort_flag);
            };
            auto issue_s = [&](int i, uint32_t u) {
                const uint64_t da = i ? dq1 : dq0, db = dk + slot_off(u);
                const uint32_t d_tm = i ? tm_s1 : tm_s0;
                if (elect_one()) {
                    if constexpr (F8) {
                        // e4m3 rows are 128 bytes: K = 32 per instruction, 32 bytes apart
#pragma unroll
                        for (int ks = 0; ks < D / 32; ++ks) {
                            const uint64_t off = (uint64_t)((ks * 32) >> 4);
                            mma_ss_f8(d_tm, da + off, db + off, idesc_qk8, ks > 0);
                        }
                    } else {
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint64_t off = (uint64_t)(((ks / 4) * kBoxBytes + (ks % 4) * 32) >> 4);
                            mma_ss(d_tm, da + off, db + off, idesc_qk, ks > 0);
                        }
                    }
                    mma_commit(&s_full[i]);
                }
                __syncwarp();
            };
            // nks: 16-key steps of the tile that hold live keys (BN / 16 but for
            // a paged sequence's last tile)
            auto issue_pv = [&](int i, uint32_t u, int j, int nks) {
                const uint64_t db = dv + slot_off(u);
                const uint32_t d_tm = i ? tm_o1 : tm_o0, p_tm = i ? tm_s1 : tm_s0;
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < BN / 16; ++ks)
                        if (ks < nks)
                        mma_ts(d_tm, p_tm + ks * 8, db + (uint64_t)((ks * 16 * 128) >> 4), idesc_pv,
                               (j > 0 || ks > 0));
                    mma_commit(&o_full[i]);
                }
                __syncwarp();
            };
            for (int r = 0; ok; ++r) {
                const int u = snake_unit(r, c, G, n_units);
                if (u < 0) break;
                UnitInfo x;
                get_unit<PAGED>(a, CAUSAL, u, x, kLaterFirst);
                const int n0 = x.n0, n1 = x.n1;
                const int nkv_max = max(n0, n1);
                if (nkv_max == 0) continue;  // a paged unit with no rows
                // tile 0's first QK^T goes out as soon as Q0 and K0 have landed;
                // Q1 (released last, loaded after K0) does not hold it back
                if (n0 > 0) ok = wait_or_abort(&q_full[0], qc0 & 1, a.err, abort_flag);
                if (ok) ok = wait_kv(ukv);
                if (!ok) break;
                tc_fence_after();
                if (n0 > 0) issue_s(0, ukv);
                if (n1 > 0) {
                    ok = wait_or_abort(&q_full[1], qc1 & 1, a.err, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(1, ukv);
                }
                if (elect_one()) {
                    mma_commit(&kv_empty[ukv % C::kStages]);
                    // a query tile with a single key tile has issued its only QK^T
                    if (n0 == 1) mma_commit(&q_empty[0]);
                    if (n1 == 1) mma_commit(&q_empty[1]);
                }
                const int n_kv_all = (x.L + BN - 1) / BN;
                for (int j = 0; j < nkv_max && ok; ++j) {
                    const uint32_t uV = ukv + 2 * j + 1, uK = ukv + 2 * j + 2;
                    ok = wait_kv(uV);
                    if (!ok) break;
                    int nks = BN / 16;
                    if (PAGED && j == n_kv_all - 1) {
                        // A paged sequence's last tile: cache slots past its end hold
                        // whatever the pool holds (NaN included) and 0 * NaN = NaN in
                        // P.V.  Issue only the 16-key steps with live keys and zero
                        // the dead V rows of the last one (masked P is ~0 there).
                        const int live = x.L - j * BN;
                        nks = (live + 15) >> 4;
                        const int dead = nks * 16 - live;  // rows live .. 16 * nks - 1
                        uint8_t *vslot = smem + C::kRingOff + (uV % C::kStages) * C::kTileBytes;
                        for (int t = lane; t < dead * 8 * C::kBoxes; t += 32) {
                            const int b = t / (dead * 8), rem = t - b * dead * 8;
                            *reinterpret_cast<uint4 *>(vslot + b * kBoxBytes + (live + rem / 8) * 128 + (rem % 8) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    bool k_ready = false;
#pragma unroll
                    for (int i = 0; i < NQ; ++i) {
                        const int ni = i ? n1 : n0;
                        if (!ok || j >= ni) continue;
                        ok = wait_or_abort(&p_full[i], ((i ? it1 : it0) + j) & 1, a.err, abort_flag);
                        if (!ok) continue;
                        tc_fence_after();
                        issue_pv(i, uV, j, nks);
                        if (j + 1 < ni) {
                            if (!k_ready) {
                                ok = wait_kv(uK);
                                if (!ok) continue;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_s(i, uK);
                            // that was the tile's last QK^T: Q_i may be reloaded once it
                            // completes, so the next unit's Q load overlaps this unit
                            if (j + 2 == ni && elect_one()) mma_commit(&q_empty[i]);
                        }
                    }
                    if (!ok) break;
                    if (elect_one()) mma_commit(&kv_empty[uV % C::kStages]);
                    if (j + 1 < nkv_max) {
                        if (!k_ready) {
                            ok = wait_kv(uK);
                            if (!ok) break;
                        }
                        if (elect_one()) mma_commit(&kv_empty[uK % C::kStages]);
                    }
                }
                ukv += 2 * nkv_max;
                it0 += n0;
                it1 += n1;
                if (n0 > 0) ++qc0;
                if (n1 > 0) ++qc1;
            }
            // every MMA issued by this thread has completed before TMEM is freed
            if (elect_one()) mma_commit(done_bar);
            __syncwarp();
            mbar_wait(done_bar, 0, nullptr);
            __syncwarp();
        }
    } else if (warp >= 10) {
        // idle warps of the producer warpgroup give their registers back
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    } else {
        // ------------------------------------------------------------ softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        const int i = warp >> 2;                 // query tile of this warpgroup
        const int quarter = warp & 3;            // TMEM lane quarter
        const int r_in = quarter * 32 + lane;    // row inside the tile
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_tm = tmem + lane_off + i * BN;
        const uint32_t o_tm = tmem + lane_off + 2 * BN + i * 128;
        bool ok = true;
        uint32_t itc = 0;        // key-tile iterations done by this query tile so far
        uint32_t stg_count = 0;  // O tiles staged by this warpgroup so far
        uint32_t ticket = 0;     // O tiles staged by both warpgroups before the current unit
        for (int rr = 0; ok; ++rr) {
            const int u = snake_unit(rr, c, G, n_units);
            if (u < 0) break;
            UnitInfo x;
            get_unit<PAGED>(a, CAUSAL, u, x, kLaterFirst);
            const int my_nkv = i ? x.n1 : x.n0;
            // the staging buffer goes to the unit's tiles in the order they
            // finish: the tile of the earlier rows first (tile 1 when causal,
            // with one key tile fewer; tile 0 otherwise); both warpgroups
            // derive the same sequence of owners
            const bool staged0 = x.n0 > 0 && (!PAGED || x.row0[0] + BM <= x.nq);
            const bool staged1 = x.n1 > 0 && (!PAGED || x.row0[1] + BM <= x.nq);
            const int first = kLaterFirst ? 1 : 0;
            const bool staged_first = first ? staged1 : staged0;
            const uint32_t my_ticket = ticket + ((i != first && staged_first) ? 1u : 0u);
            ticket += (staged0 ? 1u : 0u) + (staged1 ? 1u : 0u);
            const int tile_pos = x.pos0 + x.row0[i];  // key position of the tile's row 0
            const int row = x.row0[i] + r_in;        // query row in the sequence
            // FP8: the dequantisation scales of this query tile and of each key
            // tile fold into the softmax scale
            const float c_unit =
                (F8 && my_nkv > 0) ? a.scale_log2 * __ldg(a.q_scale + (size_t)x.head * a.nsblk + x.row0[i] / BM)
                                   : a.scale_log2;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < my_nkv; ++j) {
                ok = wait_or_abort(&s_full[i], (itc + j) & 1, a.err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[4][32];
                tmem_ld64(s_tm, sr[0], sr[1]);  // the score row in two 64-column loads
                tmem_ld64(s_tm + 64, sr[2], sr[3]);
                tmem_wait_ld();
                // visible keys: col <= lim; only key tiles reaching past the
                // tile's first row position (the causal diagonal) and the
                // sequence's last tile need masking
                const bool masked = (CAUSAL && (j + 1) * BN - 1 > tile_pos) || ((j + 1) * BN > x.L);
                if (masked) {
                    int lim = BN - 1;
                    if (CAUSAL) lim = min(lim, tile_pos + r_in - j * BN);
                    lim = min(lim, x.L - 1 - j * BN);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * cc + e > lim) sr[cc][e] = __float_as_uint(-INFINITY);
                }
                float mxa[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mxa[k] = -INFINITY;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        const int k = (e >> 3) + 4 * (cc & 1);
                        mxa[k] = max3(mxa[k], __uint_as_float(sr[cc][e]), __uint_as_float(sr[cc][e + 1]));
                        mxa[k] = max3(mxa[k], __uint_as_float(sr[cc][e + 2]), __uint_as_float(sr[cc][e + 3]));
                        mxa[k] = max3(mxa[k], __uint_as_float(sr[cc][e + 4]), __uint_as_float(sr[cc][e + 5]));
                        mxa[k] = max3(mxa[k], __uint_as_float(sr[cc][e + 6]), __uint_as_float(sr[cc][e + 7]));
                    }
                const float mx =
                    max3(max3(mxa[0], mxa[1], mxa[2]), max3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
                const float c_step = F8 ? c_unit * __ldg(a.k_scale + (size_t)x.head * a.nsblk + j) : c_unit;
                const float mx2 = mx * c_step;
                float m_ref = m;
                if (mx2 > m + kRescaleThreshold) m_ref = mx2;
                if (m_ref == -INFINITY) m_ref = 0.f;  // row with nothing visible yet
                const float alpha = ex2_approx(m - m_ref);
                const uint64_t scale2 = f2_pack(c_step, c_step);
                const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
                uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
                exp_pack_store(sr, s_tm, scale2, negm2, acc2);
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
                    ok = wait_or_abort(&o_full[i], (itc + j - 1) & 1, a.err, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld32(o_tm + 32 * cc, orr);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                        tmem_st32(o_tm + 32 * cc, orr);
                    }
                }
                m = m_ref;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[i]);
            }
            if (!ok) break;
            if (my_nkv > 0) {
                ok = wait_or_abort(&o_full[i], (itc + my_nkv - 1) & 1, a.err, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const bool live = row < x.nq;
                const size_t orow_idx = PAGED ? ((size_t)(x.qtok0 + (live ? row : 0)) * a.Hq + x.head)
                                              : ((size_t)x.head * a.N + (live ? row : 0));
                const int tile_row0 = x.row0[i];
                if (!PAGED || tile_row0 + BM <= x.nq) {
                    // The whole O tile goes, packed to bf16, into the 128B-swizzled
                    // staging buffer (one box per 64 columns), and one thread stores
                    // it with TMA (whole 128-byte row segments instead of 32 rows
                    // per store instruction; rows past the end of a dense sequence
                    // are clipped by the tensor map).  The buffer is taken in
                    // ticket order: the previous owner's store must have read it.
                    const uint32_t row_addr = smem_base + C::kStageOff + r_in * 128;
                    const bool issuer = quarter == 0 && lane == 0;
                    uint32_t pk[D / 64][32];
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        uint32_t o0[32], o1[32];
                        tmem_ld32(o_tm + 64 * h, o0);
                        tmem_ld32(o_tm + 64 * h + 32, o1);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            pk[h][e] =
                                pack_bf16x2(__uint_as_float(o0[2 * e]) * inv, __uint_as_float(o0[2 * e + 1]) * inv);
                            pk[h][16 + e] =
                                pack_bf16x2(__uint_as_float(o1[2 * e]) * inv, __uint_as_float(o1[2 * e + 1]) * inv);
                        }
                    }
                    if (my_ticket > 0) {
                        ok = wait_or_abort(&stg_free[0], (my_ticket - 1) & 1, a.err, abort_flag);
                        if (!ok) break;
                    }
#pragma unroll
                    for (int h = 0; h < D / 64; ++h)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            st_shared_v4(row_addr + h * kBoxBytes + ((ch ^ (r_in & 7)) << 4), pk[h][4 * ch],
                                         pk[h][4 * ch + 1], pk[h][4 * ch + 2], pk[h][4 * ch + 3]);
                    fence_proxy_async_smem();
                    mbar_arrive(&stg_full[i]);
                    if (issuer) {
                        ok = wait_or_abort(&stg_full[i], stg_count & 1, a.err, abort_flag);
                        if (ok) {
#pragma unroll
                            for (int h = 0; h < D / 64; ++h) {
                                if (PAGED)
                                    tma_store_2d(&tmO, smem + C::kStageOff + h * kBoxBytes, x.head * D + 64 * h,
                                                 x.qtok0 + tile_row0);
                                else
                                    tma_store_3d_hint(&tmO, smem + C::kStageOff + h * kBoxBytes, 64 * h,
                                                      tile_row0, x.head, l2_policy_evict_first());
                            }
                            bulk_commit();
                            bulk_wait_read_all();
                            mbar_arrive(&stg_free[0]);
                        }
                    }
                    ++stg_count;
                    if (!ok) break;
                } else {
                    // a paged tile that ends inside the sequence's rows: plain
                    // stores, live rows only
                    __nv_bfloat16 *orow = a.O + orow_idx * D;
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld32(o_tm + 32 * cc, orr);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv,
                                                __uint_as_float(orr[2 * e + 1]) * inv);
                        if (live) {
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * cc);
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                        }
                    }
                }
                if (live) a.LSE[orow_idx] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
                // the O reads are complete before the next unit's first PV may
                // overwrite O (ordered through p_full of that unit)
                tc_fence_before();
            }
            itc += my_nkv;
        }
        // the staged O stores are complete before the CTA exits
        if (quarter == 0 && lane == 0) bulk_wait_all();
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

// 2-D bf16 tensor map: `rows` rows of `inner` elements (row pitch
// `pitch_elems`), box 64 x box_rows, 128B swizzle.
bool make_map_2d(CUtensorMap *m, const void *base, long long inner, long long rows, long long pitch_elems,
                 int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch_elems * 2};
    cuuint32_t box[2] = {kBoxCols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
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
        if (cudaFuncSetAttribute(prefill_bf16_kernel<D, CAUSAL, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    CUtensorMap tq, tk, tv, to;
    const int BH = p.B * p.H;
    if (!make_map(&tq, p.Q, p.N, D, BH) || !make_map(&tk, p.K, p.N, D, BH) || !make_map(&tv, p.V, p.N, D, BH) ||
        !make_map(&to, p.O, p.N, D, BH))
        return ATTN_ECUDA;
    PrefillArgs a = {};
    a.O = static_cast<__nv_bfloat16 *>(p.O);
    a.LSE = p.LSE;
    a.err = p.err_flag;
    a.N = p.N;
    a.BH = BH;
    a.nblk = (p.N + NQ * BM - 1) / (NQ * BM);
    a.scale_log2 = p.scale * 1.4426950408889634f;
    static int sm_count[64] = {0};
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    // persistent: one CTA per SM (the shared-memory footprint allows no more),
    // each walking its units in snake order
    const long long units = (long long)a.nblk * BH;
    const int grid = (int)(units < sm_count[dev] ? units : sm_count[dev]);
    prefill_bf16_kernel<D, CAUSAL, false><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

template <int D>
attn_status launch_paged_t(const PagedPrefillLaunch &p, cudaStream_t stream) {
    using C = Cfg<D>;
    static bool attr_set[64] = {false};
    static int sm_count[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(prefill_bf16_kernel<D, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    CUtensorMap tq, tk, tv, to;
    const long long cache_rows = (long long)p.num_blocks * p.Hkv * p.block_size;
    if (!make_map_2d(&tq, p.q, (long long)p.Hq * D, p.total_q, (long long)p.Hq * D, BM) ||
        !make_map_2d(&tk, p.k_cache, D, cache_rows, D, p.block_size) ||
        !make_map_2d(&tv, p.v_cache, D, cache_rows, D, p.block_size) ||
        !make_map_2d(&to, p.O, (long long)p.Hq * D, p.total_q, (long long)p.Hq * D, BM))
        return ATTN_ECUDA;
    PrefillArgs a = {};
    a.O = static_cast<__nv_bfloat16 *>(p.O);
    a.LSE = p.LSE;
    a.err = p.err_flag;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.cu_q = p.cu_q;
    a.seq_lens = p.seq_lens;
    a.block_table = p.block_table;
    a.S = p.num_seqs;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.max_blocks = p.max_blocks;
    a.num_blocks = p.num_blocks;
    a.block_size = p.block_size;
    a.nqb = (p.max_q_per_seq + NQ * BM - 1) / (NQ * BM);
    a.total_q = p.total_q;
    const long long units = (long long)a.nqb * a.S * a.Hq;
    if (units == 0) return ATTN_OK;
    const int grid = (int)(units < sm_count[dev] ? units : sm_count[dev]);
    prefill_bf16_kernel<D, true, true><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

// [B*H, N, d] e4m3 (bytes) viewed as a 3-D tensor map, box 128 x 128 x 1
// (one 128-byte row per box row), 128B swizzle.
bool make_map_u8(CUtensorMap *m, const void *base, int N, int d, int BH) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)N * d};
    cuuint32_t box[3] = {128, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool CAUSAL>
attn_status launch_fp8_t(const Fp8Launch &p, cudaStream_t stream) {
    constexpr int D = 128;
    using C = Cfg<D>;
    static bool attr_set[64] = {false};
    static int sm_count[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(prefill_bf16_kernel<D, CAUSAL, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    const int BH = p.B * p.H;
    CUtensorMap tq, tk, tv, to;
    if (!make_map_u8(&tq, p.q8, p.N, D, BH) || !make_map_u8(&tk, p.k8, p.N, D, BH) ||
        !make_map(&tv, p.V, p.N, D, BH) || !make_map(&to, p.O, p.N, D, BH))
        return ATTN_ECUDA;
    PrefillArgs a = {};
    a.O = static_cast<__nv_bfloat16 *>(p.O);
    a.LSE = p.LSE;
    a.err = p.err_flag;
    a.N = p.N;
    a.BH = BH;
    a.nblk = (p.N + NQ * BM - 1) / (NQ * BM);
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.q_scale = p.q_scale;
    a.k_scale = p.k_scale;
    a.nsblk = (p.N + BM - 1) / BM;
    const long long units = (long long)a.nblk * BH;
    const int grid = (int)(units < sm_count[dev] ? units : sm_count[dev]);
    prefill_bf16_kernel<D, CAUSAL, false, true><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace

bool make_tensor_map_2d_bf16(CUtensorMap *m, const void *base, long long inner, long long rows, long long pitch_elems,
                             int box_rows) {
    return make_map_2d(m, base, inner, rows, pitch_elems, box_rows);
}

attn_status launch_prefill_fp8(const Fp8Launch &p, cudaStream_t stream) {
    return p.causal ? launch_fp8_t<true>(p, stream) : launch_fp8_t<false>(p, stream);
}

attn_status launch_paged_prefill(const PagedPrefillLaunch &p, cudaStream_t stream) {
    return p.d == 128 ? launch_paged_t<128>(p, stream) : launch_paged_t<64>(p, stream);
}

attn_status launch_prefill_bf16(const DenseLaunch &p, cudaStream_t stream) {
    if (p.d == 128) return p.causal ? launch_t<128, true>(p, stream) : launch_t<128, false>(p, stream);
    return p.causal ? launch_t<64, true>(p, stream) : launch_t<64, false>(p, stream);
}

}  // namespace osp
