// decode_paged.cu -- paged-KV decode for sm_100a: one query token per
// sequence, keys/values gathered through a per-sequence block table.
//
// Method (pages): "第 2 章核心模块：FlashAttention-2 与 PagedAttention 实现解析"
// section 2.2 -- for each logical block look up the physical block, fetch
// only that block's K/V, score it and merge into the running max/sum;
// section 2.1 -- the incremental normalisation (running max m, running sum l,
// correct the accumulated O).  "一文掌握大模型推理加速：FlashAttention与
// PagedAttention技术详解" section 三 核心原理 -- fixed blocks of 16 or 32
// tokens, contiguous logical / non-contiguous physical blocks.
//
// B200 design (HBM-bound: ~1 flop per byte):
//   1. plan kernel  -- one CTA scans seq_lens into per-sequence split offsets
//                      (split size fixed by the host from the sizes only),
//                      zeroes the work counter and the per-(sequence, head)
//                      completion counters, and writes the result of empty or
//                      invalid-length sequences (O = 0, LSE = -inf).
//   2. split kernel -- persistent, one CTA per SM, every warp an independent
//                      worker, launched as a programmatic dependent of the
//                      plan.  A warp takes (sequence, split, head) items from
//                      an atomic counter and streams the split's 16-token K
//                      and V tiles (4 KiB each, contiguous inside a block)
//                      into its own ring of shared-memory slots with 1-D bulk
//                      async copies completing on per-slot mbarriers.  Math
//                      reads the slots with 16-byte vector loads: a half-warp
//                      holds one 128-wide row (8 dims per lane), q.k is reduced
//                      with warp shuffles, and the online-softmax update is
//                      applied once per tile.  A sequence with one split
//                      writes O and LSE directly; otherwise each split writes
//                      a normalised partial O and its log2-sum-exp, and the
//                      warp that completes the last split of a (sequence,
//                      head) merges them in split order:
//                      LSE = log sum_p exp(LSE_p), O = sum_p e^{LSE_p-LSE} O_p.
// Every arithmetic order depends only on logical token positions (which warp
// runs a split, or merges, changes nothing), so moving blocks to other
// physical ids gives bit-identical results.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "launch.h"
#include "ptx.cuh"

namespace osp {
namespace {

constexpr int kD = 128;                         // head dim supported here
constexpr int kTileTok = 16;                    // tokens per pipeline tile
constexpr int kTileBytes = kTileTok * kD * 2;   // 4 KiB of K (or of V)
constexpr int kStages = 2;                      // ring slots per worker
constexpr int kSlotBytes = 2 * kTileBytes;      // K tile + V tile
constexpr int kMaxSmemSeqs = 4096;  // split offsets staged in shared memory up to this many sequences
// Workers per CTA: 12 for one query head per key/value head, fewer for
// larger groups (each worker holds G query rows, accumulators and maxima).
template <int G>
struct Warps {
    static constexpr int value = G >= 4 ? 8 : 12;
};
template <int W>
constexpr int smem_bytes() {
    return W * kStages * kSlotBytes + W * kStages * 8 + (kMaxSmemSeqs + 1) * 4 + 64;
}

struct DecodeArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *block_table;
    const int32_t *seq_lens;
    __nv_bfloat16 *O;
    float *LSE;
    int32_t *err;
    // workspace views
    int32_t *counter;     // [1]
    int32_t *item_start;  // [num_seqs + 1] prefix sum of splits per sequence
    int32_t *done_cnt;    // [num_seqs, H] splits finished per (sequence, head)
    int32_t *seq_bad;     // [num_seqs] nonzero: a block-table entry was out of range
    float *part_lse;      // [num_seqs, H, max_splits] log2 units
    float *part_o;        // [num_seqs, H, max_splits, d] normalised
    int num_seqs, H, num_blocks, max_blocks, block_size, split_tokens, max_splits;
    int Hkv;              // key/value heads; H (query heads) = Hkv * G
    float scale_log2;     // scale * log2(e)
};

__device__ __forceinline__ bool seq_len_ok(int L, const DecodeArgs &a) {
    return L >= 0 && (long long)L <= (long long)a.max_blocks * a.block_size;
}

// ------------------------------------------------------------------ plan

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__global__ void __launch_bounds__(1024) decode_plan_kernel(DecodeArgs a) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    pdl_launch_dependents();  // the split kernel may start its prologue now
    if (tid == 0) {
        carry = 0;
        *a.counter = 0;
    }
    for (int i = tid; i < a.num_seqs * a.H; i += 1024) a.done_cnt[i] = 0;
    // sequences with no split (empty, or an invalid length): their rows are
    // written here, one warp per such sequence
    for (int s = wid; s < a.num_seqs; s += 32) {
        const int L = a.seq_lens[s];
        if (L > 0 && seq_len_ok(L, a)) continue;
        if (lane == 0) {
            a.seq_bad[s] = 0;
            if (!seq_len_ok(L, a) && a.err) atomicOr(a.err, ATTN_DEVERR_SEQ_LEN);
        }
        for (int e = lane; e < a.H * (kD / 8); e += 32)
            reinterpret_cast<uint4 *>(a.O + (size_t)s * a.H * kD)[e] = make_uint4(0u, 0u, 0u, 0u);
        for (int h = lane; h < a.H; h += 32) a.LSE[(size_t)s * a.H + h] = -INFINITY;
    }
    for (int i = tid; i < a.num_seqs; i += 1024) a.seq_bad[i] = 0;
    __syncthreads();
    for (int base = 0; base < a.num_seqs; base += 1024) {
        const int s = base + tid;
        int n = 0;
        if (s < a.num_seqs) {
            const int L = a.seq_lens[s];
            if (seq_len_ok(L, a)) n = (L + a.split_tokens - 1) / a.split_tokens;
        }
        int x = n;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int w = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_tot[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int excl = carry + (wid ? warp_tot[wid - 1] : 0) + x - n;
        if (s < a.num_seqs) a.item_start[s] = excl;
        __syncthreads();
        if (tid == 1023) carry = excl + n;
        __syncthreads();
    }
    if (tid == 0) a.item_start[a.num_seqs] = carry;
}

// ------------------------------------------------------------------ split

constexpr float kLn2 = 0.69314718055994530942f;

// One unit of work: tokens [tok0, tok1) of sequence s, key/value head h
// (split p); with a group of G query heads per key/value head it serves query
// heads h*G .. h*G+G-1.  Everything is warp-uniform except tbl0/tbl1/qv: lane
// l holds the physical ids of the item's blocks l and 32 + l, and (G == 1)
// 16 bytes (8 dims) of the q row.
struct Item {
    int s, h, p, tok0, tok1, nt;  // nt: 16-token tiles (0: no item)
    int tbl0, tbl1;
    uint4 qv;
};

// Take the next item from the work counter (all lanes; lane 0 does the
// atomic).  Loads the item's block-table entries and q row into registers
// now, so neither is a dependent load later.
template <int G>
__device__ __forceinline__ void fetch_item(const DecodeArgs &a, const int32_t *starts, int total, int lane,
                                           int &s_hint, Item &it) {
    int idx = 0;
    if (lane == 0) idx = atomicAdd(a.counter, 1);
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= total) {
        it.nt = 0;
        return;
    }
    const int k = idx / a.Hkv;
    it.h = idx - k * a.Hkv;
    // sequence holding split k: starts[s] <= k < starts[s + 1]
    int lo = 0, hi = a.num_seqs - 1;
    if (starts[s_hint] <= k && k < starts[s_hint + 1]) {
        lo = s_hint;
    } else {
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= k) lo = mid; else hi = mid - 1;
        }
    }
    s_hint = it.s = lo;
    it.p = k - starts[lo];
    it.tok0 = it.p * a.split_tokens;
    // independent loads: the length, the split's block ids (up to 64, read
    // within the table row whatever the length), the q row
    const int L = a.seq_lens[lo];
    const int lb0 = it.tok0 / a.block_size;
    const int room = a.max_blocks - lb0;
    const int32_t *row = a.block_table + (size_t)lo * a.max_blocks + lb0;
    const int t0 = lane < room ? __ldg(row + lane) : -1;
    const int t1 = lane + 32 < room ? __ldg(row + 32 + lane) : -1;
    if (G == 1) it.qv = *reinterpret_cast<const uint4 *>(a.q + ((size_t)lo * a.H + it.h) * kD + 8 * (lane & 15));
    it.tok1 = min(L, it.tok0 + a.split_tokens);
    it.nt = (it.tok1 - it.tok0 + kTileTok - 1) / kTileTok;
    const int nblk = (it.tok1 - it.tok0 + a.block_size - 1) / a.block_size;  // <= 64 by the split choice
    it.tbl0 = lane < nblk ? t0 : -1;
    it.tbl1 = lane + 32 < nblk ? t1 : -1;
}

// Physical block of tile t of the item (all lanes; -1 when out of range).
__device__ __forceinline__ int tile_block(const DecodeArgs &a, const Item &it, int t) {
    const int bi = (t * kTileTok) / a.block_size;  // tok0 is a multiple of block_size
    const int v = __shfl_sync(0xffffffffu, bi < 32 ? it.tbl0 : it.tbl1, bi & 31);
    return (v >= 0 && v < a.num_blocks) ? v : -1;
}

// Lane 0: start the copies of tile t of `it` into `slot` (or, for a block
// outside the pool, complete the slot's phase without touching memory).
__device__ __forceinline__ void issue_tile(const DecodeArgs &a, uint8_t *slots, uint64_t *full, int slot,
                                           const Item &it, int t, int phys) {
    uint64_t *bar = full + slot;
    if (phys < 0) {
        if (a.err) atomicOr(a.err, ATTN_DEVERR_BLOCK_TABLE);
        mbar_arrive(bar);
        return;
    }
    const int tok = it.tok0 + t * kTileTok;
    const size_t off = (((size_t)phys * a.Hkv + it.h) * a.block_size + (tok % a.block_size)) * kD;
    uint8_t *dst = slots + slot * kSlotBytes;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, kSlotBytes);
    bulk_g2s(dst, a.k_cache + off, kTileBytes, bar);
    bulk_g2s(dst + kTileBytes, a.v_cache + off, kTileBytes, bar);
}

// Final bf16 row of O (o * inv_l, or zeros when o is null) and its LSE.
// Lanes of half 0 hold dims 8*li .. 8*li+7.
__device__ __forceinline__ void final_store(const DecodeArgs &a, size_t sh, int li, int half, int lane,
                                            const float *o, float inv_l, float lse) {
    if (half == 0) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (o) {
            w.x = pack_bf16x2(o[0] * inv_l, o[1] * inv_l);
            w.y = pack_bf16x2(o[2] * inv_l, o[3] * inv_l);
            w.z = pack_bf16x2(o[4] * inv_l, o[5] * inv_l);
            w.w = pack_bf16x2(o[6] * inv_l, o[7] * inv_l);
        }
        *reinterpret_cast<uint4 *>(a.O + sh * kD + 8 * li) = w;
    }
    if (lane == 0) a.LSE[sh] = lse;
}

// Output of a finished item: the final row for a one-split sequence, else a
// partial; the warp completing the last split of (s, h) merges in split order.
__device__ __forceinline__ void finish_item(const DecodeArgs &a, int s, int hq, int p, int lane, float m, float l,
                                            float (&o)[8], bool saw_bad) {
    const int half = lane >> 4, li = lane & 15;
    l += __shfl_xor_sync(0xffffffffu, l, 16);
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] += __shfl_xor_sync(0xffffffffu, o[c], 16);
    const int nsplit = a.item_start[s + 1] - a.item_start[s];  // (L2-resident, once per item)
    const size_t sh = (size_t)s * a.H + hq;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    if (nsplit == 1) {
        if (saw_bad)
            final_store(a, sh, li, half, lane, nullptr, 0.f, -INFINITY);
        else
            final_store(a, sh, li, half, lane, o, inv_l, l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY);
        return;
    }
    const size_t pidx = sh * a.max_splits + p;
    if (half == 0) {
        float4 *dst = reinterpret_cast<float4 *>(a.part_o + pidx * kD + 8 * li);
        dst[0] = make_float4(o[0] * inv_l, o[1] * inv_l, o[2] * inv_l, o[3] * inv_l);
        dst[1] = make_float4(o[4] * inv_l, o[5] * inv_l, o[6] * inv_l, o[7] * inv_l);
    }
    if (lane == 0) {
        a.part_lse[pidx] = l > 0.f ? m + __log2f(l) : -INFINITY;
        if (saw_bad) atomicOr(a.seq_bad + s, 1);
    }
    __threadfence();  // partials (and the bad mark) before the completion count
    __syncwarp();
    int last = 0;
    if (lane == 0) last = (atomicAdd(a.done_cnt + sh, 1) == nsplit - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    if (__ldcg(a.seq_bad + s)) {
        final_store(a, sh, li, half, lane, nullptr, 0.f, -INFINITY);
        return;
    }
    const float *plse = a.part_lse + sh * a.max_splits;
    float M = -INFINITY;
    for (int q = 0; q < nsplit; ++q) M = fmaxf(M, __ldcg(plse + q));
    float tot = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < nsplit; ++q) {
        const float w = ex2_approx(__ldcg(plse + q) - M);
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.part_o + (sh * a.max_splits + q) * kD) + lane);
        tot += w;
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(a.O + sh * kD + 4 * lane) = packed;
    if (lane == 0) a.LSE[sh] = tot > 0.f ? (M + __log2f(tot)) * kLn2 : -INFINITY;
}

template <int G>
__global__ void __launch_bounds__(Warps<G>::value * 32, 1) decode_split_kernel(DecodeArgs a) {
    constexpr int kWarps = Warps<G>::value;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint8_t *slots = smem + (size_t)wid * kStages * kSlotBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kWarps * kStages * kSlotBytes) + wid * kStages;
    if (lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(full + i, 1);
        fence_barrier_init();
    }
    __syncwarp();
    const int half = lane >> 4, li = lane & 15;
    pdl_wait();  // the plan kernel's writes are visible from here on
    // per-sequence split offsets, staged in shared memory when they fit
    const int32_t *starts = a.item_start;
    if (a.num_seqs <= kMaxSmemSeqs) {
        int32_t *st = reinterpret_cast<int32_t *>(smem + kWarps * kStages * kSlotBytes + kWarps * kStages * 8);
        for (int i = threadIdx.x; i <= a.num_seqs; i += blockDim.x) st[i] = a.item_start[i];
        __syncthreads();
        starts = st;
    }
    const int total = starts[a.num_seqs] * a.Hkv;
    int s_hint = 0;

    // The warp is a stream of 16-token tiles over consecutive items: the
    // producer (lane 0's copies) runs kStages tiles ahead of the consumer,
    // crossing into the next item (cur -> nxt) so the ring never drains.
    Item cur, nxt;
    fetch_item<G>(a, starts, total, lane, s_hint, cur);
    bool have_nxt = false, exhausted = (cur.nt == 0);
    int pq = 0, pt = 0;           // producer: item (0 cur, 1 nxt) and next tile
    uint32_t gi = 0, gc = 0;      // tiles issued / consumed by this warp
    bool dead = false;

    auto produce = [&]() -> bool {
        for (;;) {
            const int pnt = pq ? nxt.nt : cur.nt;
            if (pt < pnt) {
                const int phys = pq ? tile_block(a, nxt, pt) : tile_block(a, cur, pt);
                if (lane == 0) issue_tile(a, slots, full, gi % kStages, pq ? nxt : cur, pt, phys);
                ++pt;
                ++gi;
                return true;
            }
            if (pq == 1 || exhausted) return false;
            fetch_item<G>(a, starts, total, lane, s_hint, nxt);
            if (nxt.nt == 0) {
                exhausted = true;
                return false;
            }
            have_nxt = true;
            pq = 1;
            pt = 0;
        }
    };

    if (!exhausted) {
        while (gi - gc < (uint32_t)kStages && produce()) {
        }
    }
    while (!exhausted || cur.nt > 0) {
        if (cur.nt == 0) break;
        // query rows of the group, 8 dims per lane, pre-scaled into log2 units
        float qf[G][8];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uint4 qv;
            if (G == 1)
                qv = cur.qv;
            else
                qv = *reinterpret_cast<const uint4 *>(a.q + ((size_t)cur.s * a.H + cur.h * G + g) * kD + 8 * li);
            const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                qf[g][2 * c] = bf16lo(w[c]) * a.scale_log2;
                qf[g][2 * c + 1] = bf16hi(w[c]) * a.scale_log2;
            }
        }
        float m[G], l[G], o[G][8];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) o[g][c] = 0.f;
        }
        bool saw_bad = false;
        for (int t = 0; t < cur.nt; ++t) {
            const int slot = gc % kStages;
            if (!mbar_wait(full + slot, (gc / kStages) & 1u, a.err)) {
                dead = true;
                break;
            }
            const int tok = cur.tok0 + t * kTileTok;
            const bool tile_ok = tile_block(a, cur, t) >= 0;
            saw_bad |= !tile_ok;
            if (tile_ok) {
                const uint8_t *kt = slots + slot * kSlotBytes;
                const uint8_t *vt = kt + kTileBytes;
                // scores of all G query heads: each K row is read and converted once
                float sc[G][8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 2 * i + half;
                    const uint4 kv = *reinterpret_cast<const uint4 *>(kt + r * (kD * 2) + li * 16);
                    const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
                    float kf[8];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        kf[2 * c] = bf16lo(w[c]);
                        kf[2 * c + 1] = bf16hi(w[c]);
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float acc = 0.f;
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc = fmaf(qf[g][c], kf[c], acc);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                        sc[g][i] = (tok + r < cur.tok1) ? acc : -INFINITY;
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float mt = sc[g][0];
#pragma unroll
                    for (int i = 1; i < 8; ++i) mt = fmaxf(mt, sc[g][i]);
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                    const float m_new = fmaxf(m[g], mt);
                    const float alpha = ex2_approx(m[g] - m_new);
                    float psum = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sc[g][i] = ex2_approx(sc[g][i] - m_new);
                        psum += sc[g][i];
                    }
                    l[g] = l[g] * alpha + psum;
#pragma unroll
                    for (int c = 0; c < 8; ++c) o[g][c] *= alpha;
                    m[g] = m_new;
                }
                // P V for all G heads: each V row is read and converted once
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 2 * i + half;
                    if (tok + r < cur.tok1) {
                        const uint4 vv = *reinterpret_cast<const uint4 *>(vt + r * (kD * 2) + li * 16);
                        const uint32_t w[4] = {vv.x, vv.y, vv.z, vv.w};
                        float vf[8];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            vf[2 * c] = bf16lo(w[c]);
                            vf[2 * c + 1] = bf16hi(w[c]);
                        }
#pragma unroll
                        for (int g = 0; g < G; ++g)
#pragma unroll
                            for (int c = 0; c < 8; ++c) o[g][c] = fmaf(sc[g][i], vf[c], o[g][c]);
                    }
                }
            }
            ++gc;
            __syncwarp();  // every lane is done with the slot before it is refilled
            if (gi - gc < (uint32_t)kStages) produce();
        }
        if (dead) break;
#pragma unroll
        for (int g = 0; g < G; ++g) finish_item(a, cur.s, cur.h * G + g, cur.p, lane, m[g], l[g], o[g], saw_bad);
        if (!have_nxt) break;
        cur = nxt;
        have_nxt = false;
        pq = 0;
        while (gi - gc < (uint32_t)kStages && produce()) {
        }
    }

    // after a timeout: wait (bounded) for this warp's copies still in flight
    // so no bulk copy lands in shared memory after the CTA has exited
    if (dead && lane == 0) {
        for (uint32_t g = gc; g < gi; ++g) mbar_wait(full + g % kStages, (g / kStages) & 1u, nullptr);
    }
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
    size_t counter, item_start, done_cnt, seq_bad, part_lse, part_o, total;
};

WsLayout ws_layout(int num_seqs, int H, int max_splits) {
    WsLayout w;
    w.counter = 0;
    w.item_start = 256;
    w.done_cnt = align_up(w.item_start + sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
    w.seq_bad = align_up(w.done_cnt + sizeof(int32_t) * (size_t)num_seqs * H, 256);
    w.part_lse = align_up(w.seq_bad + sizeof(int32_t) * (size_t)num_seqs, 256);
    w.part_o = align_up(w.part_lse + sizeof(float) * (size_t)num_seqs * H * max_splits, 256);
    w.total = align_up(w.part_o + sizeof(float) * (size_t)num_seqs * H * max_splits * kD, 256);
    return w;
}

}  // namespace

int decode_split_tokens(int num_seqs, int H, int d, int max_blocks, int block_size) {
    (void)d;
    const long long max_len = (long long)max_blocks * block_size;
    const long long work = (long long)num_seqs * H * max_len;
    long long split = 256;
    // larger splits for large problems (bounded workspace), at most 64 blocks
    // per split (the kernel keeps a split's block ids in two registers per lane)
    while (split < max_len && work / split > 65536 && split * 2 <= 64LL * block_size) split <<= 1;
    return (int)split;
}

int decode_max_splits(int num_seqs, int H, int d, int max_blocks, int block_size) {
    const long long max_len = (long long)max_blocks * block_size;
    const int split = decode_split_tokens(num_seqs, H, d, max_blocks, block_size);
    return (int)((max_len + split - 1) / split);
}

size_t decode_workspace_bytes(int num_seqs, int H, int d, int max_blocks, int block_size) {
    const int ms = decode_max_splits(num_seqs, H, d, max_blocks, block_size);
    return ws_layout(num_seqs, H, ms < 1 ? 1 : ms).total;
}

template <int G>
attn_status launch_split(const DecodeArgs &a, int dev, int sms, cudaStream_t stream) {
    constexpr int W = Warps<G>::value;
    static bool attr_set[64] = {false};
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(decode_split_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes<W>()) != cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    // the split kernel is a programmatic dependent of the plan: its launch and
    // barrier set-up overlap the plan; griddepcontrol.wait orders the data
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(W * 32);
    cfg.dynamicSmemBytes = smem_bytes<W>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_split_kernel<G>, a) == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

attn_status launch_paged_decode(const DecodeLaunch &p, cudaStream_t stream) {
    static int sm_count[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ECUDA;
    if (dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    const int G = p.H / p.Hkv;
    DecodeArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(p.q);
    a.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    a.block_table = p.block_table;
    a.seq_lens = p.seq_lens;
    a.O = static_cast<__nv_bfloat16 *>(p.O);
    a.LSE = p.LSE;
    a.err = p.err_flag;
    a.num_seqs = p.num_seqs;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.num_blocks = p.num_blocks;
    a.max_blocks = p.max_blocks;
    a.block_size = p.block_size;
    a.split_tokens = decode_split_tokens(p.num_seqs, p.H, p.d, p.max_blocks, p.block_size);
    a.max_splits = decode_max_splits(p.num_seqs, p.H, p.d, p.max_blocks, p.block_size);
    if (a.max_splits < 1) a.max_splits = 1;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    const WsLayout w = ws_layout(p.num_seqs, p.H, a.max_splits);
    uint8_t *ws = static_cast<uint8_t *>(p.workspace);
    a.counter = reinterpret_cast<int32_t *>(ws + w.counter);
    a.item_start = reinterpret_cast<int32_t *>(ws + w.item_start);
    a.done_cnt = reinterpret_cast<int32_t *>(ws + w.done_cnt);
    a.seq_bad = reinterpret_cast<int32_t *>(ws + w.seq_bad);
    a.part_lse = reinterpret_cast<float *>(ws + w.part_lse);
    a.part_o = reinterpret_cast<float *>(ws + w.part_o);

    decode_plan_kernel<<<1, 1024, 0, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ECUDA;
    switch (G) {
        case 1: return launch_split<1>(a, dev, sm_count[dev], stream);
        case 2: return launch_split<2>(a, dev, sm_count[dev], stream);
        case 4: return launch_split<4>(a, dev, sm_count[dev], stream);
        case 8: return launch_split<8>(a, dev, sm_count[dev], stream);
    }
    return ATTN_EUNSUPPORTED;
}

}  // namespace osp
