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
//   Grouped query heads (G = 4, 8, and groups of 8 above) take a third
//   route, described at decode_mma_kernel: warp tensor-core MMAs per 16-key
//   tile, a balanced static schedule of equal tile runs planned inside the
//   kernel, a producer warp refilling each math warp's ring, and
//   decode_merge_kernel for the rows the runs cut.
// Every arithmetic order depends only on the lengths and sizes (which warp
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
    int32_t *slot_bad;    // [partial slots] grouped kernel: the slot's segment met a bad block id
    float *part_lse;      // [num_seqs, H, max_splits] log2 units
    float *part_o;        // [num_seqs, H, max_splits, d] normalised
    int num_seqs, H, num_blocks, max_blocks, block_size, split_tokens, max_splits;
    int Hkv;              // key/value heads of the item space; H (query heads) = Hkv * G
    int kv_heads;         // key/value heads of the cache (= Hkv, or Hkv / kv_div)
    int kv_div;           // groups above 8 run as kv_div groups of 8 per cache head
    int bs_shift;         // log2(block_size)
    float scale_log2;     // scale * log2(e)
    int fused_plan;       // grouped kernel: every CTA computes the plan itself (no plan kernel)
    int sched_w;          // grouped kernel: schedule width (math warps of the launch, at most kMaxWorkers)
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

__device__ __forceinline__ void merge_row(const DecodeArgs &a, int s, size_t sh, int nsplit, int lane);

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
    merge_row(a, s, sh, nsplit, lane);
}

// The final row of (sequence s, query head) sh from its nsplit normalised
// partials, in split order (all lanes; lane l owns dims 4l .. 4l+3).
__device__ __forceinline__ void merge_row(const DecodeArgs &a, int s, size_t sh, int nsplit, int lane) {
    if (__ldcg(a.seq_bad + s)) {
        *reinterpret_cast<uint2 *>(a.O + sh * kD + 4 * lane) = make_uint2(0u, 0u);
        if (lane == 0) a.LSE[sh] = -INFINITY;
        return;
    }
    const float *plse = a.part_lse + sh * a.max_splits;
    float M = -INFINITY;
#pragma unroll 4
    for (int q = 0; q < nsplit; ++q) M = fmaxf(M, __ldcg(plse + q));
    float tot = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
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

// ------------------------------------------------------------------ grouped heads on tensor cores
//
// For G >= 4 query heads per key/value head the per-row shuffle reductions
// above bound the kernel, not HBM.  This variant computes each 16-key tile
// with warp-level tensor core MMAs (m16n8k16, bf16 in, fp32 accumulate):
// S = Q K^T with the G query rows padded to 16, then O^T += V^T P^T, where
// the query heads are the product's 8 columns (no padding for G = 8) and
// P^T's fragments are exactly the S accumulators a lane holds.  K/V tiles
// arrive by TMA in 128-byte-swizzled boxes so that the ldmatrix fragment
// loads are conflict-free.
//
// Work is not taken from a queue: every (sequence, key/value head) row has
// ceil(L / 16) tiles, the rows are laid end to end (sequence-major), and
// worker w of nw takes tiles [floor(w T / nw), floor((w + 1) T / nw)) of
// that line for T tiles in all, with nw = min(W, max(1, floor(T / 8))) and
// W the launch's math warps (at most kMaxWorkers): every warp has a run,
// the runs differ by at most one tile, and none is shorter than 8 tiles
// (128 keys) unless T is.  Every worker then streams the same number of
// bytes whatever the length mix; a worker's run crosses row boundaries as
// it comes.  The worker holding tile x is floor(((x + 1) nw - 1) / T).  A
// row cut by worker boundaries into n segments gets n partials, stored at
// slots worker + row (so one row's slots are consecutive, and all slots fit
// in nw + rows), merged by decode_merge_kernel.  The plan depends on the
// lengths, the sizes and the launch's width only, so results do not depend
// on the physical block ids or on which warp ran a worker.
//
// A CTA is 8 math warps and one producer warp (in a warpgroup of its own,
// the register split moving registers to the math warps).  Lane c of the
// producer walks math warp c's schedule tile by tile, reads the block ids
// one tile ahead, and issues each tile's TMA copies into warp c's 2-slot ring
// as soon as the warp releases the slot (full / empty mbarriers per slot),
// so the math warps only wait, compute and release.

constexpr int kCons = 8;                          // math warps per CTA
constexpr int kMmaThreads = (kCons + 4) * 32;     // + the producer's warpgroup
constexpr int kConsRegs = 224, kProdRegs = 56;    // 256 x 224 + 128 x 56 = 384 x 168
constexpr int kMaxWorkers = 148 * 10;             // schedule width bound (the workspace holds its slots)
constexpr int kMinTiles = 8;                      // shortest worker run: 128 keys
constexpr float kLazyLog2 = 8.f;  // rescale only when the max grows by more than 2^8
constexpr int kScratchBytes = 8 * kD * 4;  // per math warp: up to 8 unnormalised O rows (fp32)
constexpr int kRingBytes = kCons * kStages * kSlotBytes;
constexpr int kBarOff = kRingBytes + kCons * kScratchBytes;    // full[kCons][2], empty[kCons][2]
constexpr int kBadOff = kBarOff + 2 * kCons * kStages * 8;      // slot_bad[kCons][2] (int)
constexpr int kStartsOff = kBadOff + kCons * kStages * 4;
constexpr int kMmaSmem = kStartsOff + (kMaxSmemSeqs + 1) * 4 + 1024;
static_assert(kConsRegs * kCons * 32 + kProdRegs * 128 <= 168 * kMmaThreads, "register split");

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A B + D, m16n8k16, A row-major bf16, B column-major bf16, fp32 D.
__device__ __forceinline__ void mma_bf16_4(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The same with rows 8..15 of A zero (the padding of the query group).
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk c (0..15: dims 8c..8c+7) of tile row r in a
// slot half (two 64-column boxes of 16 rows, 128-byte swizzle).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 3) * 2048 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Non-blocking probe of an mbarrier phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// One piece of a math warp's run: tiles of one row (sequence s, key/value
// head h), the whole of it inside one segment (the part of the row in one
// worker's run).
struct SegItem {
    int s, h, tok0, tok1, nt;  // tokens [tok0, tok1), nt 16-token tiles (0: none)
    int w;                     // the worker whose run holds the item
    bool first, last;          // the item opens / closes its segment
};

// Where a worker's walk stands: worker w, its run [x, x_end) still to go.
struct SchedPos {
    int w;
    long long x, x_begin, x_end;
};

// The sequence whose rows hold tile x: Hkv starts[s] <= x < Hkv starts[s + 1]
// (starts: tiles before each sequence; empty sequences share a start).
__device__ __forceinline__ int seq_of_tile(const DecodeArgs &a, const int32_t *starts, long long x, int s_hint) {
    const int c = (int)(x / a.Hkv);
    if (starts[s_hint] <= c && c < starts[s_hint + 1]) return s_hint;
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (starts[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// The schedule: T tiles over nw workers in runs differing by at most one
// tile.
struct Sched {
    long long T, nw;
};

__host__ __device__ __forceinline__ long long sched_nw(long long T, int W) {
    const long long by_len = T / kMinTiles;
    return by_len < 1 ? 1 : (by_len < W ? by_len : W);
}

// first tile of worker w's run (w in [0, nw]; w = nw gives T)
__device__ __forceinline__ long long run_begin(const Sched &sc, long long w) { return w * sc.T / sc.nw; }

// the worker whose run holds tile x (x in [0, T))
__device__ __forceinline__ long long worker_of(const Sched &sc, long long x) { return ((x + 1) * sc.nw - 1) / sc.T; }

// Start worker run ps.w + stride (false: none left).
__device__ __forceinline__ bool next_worker(SchedPos &ps, const Sched &sc, int stride) {
    ps.w += stride;
    if (ps.w >= sc.nw) return false;
    ps.x_begin = ps.x = run_begin(sc, ps.w);
    ps.x_end = run_begin(sc, ps.w + 1);
    return true;
}

// The next item of a math warp (warp-uniform): the rest of the current row
// inside the current worker's run, then the next worker (w + stride).
__device__ __forceinline__ void next_seg_item(const DecodeArgs &a, const int32_t *starts, const Sched &sc, int stride,
                                              int &s_hint, SchedPos &ps, SegItem &it) {
    if (ps.x >= ps.x_end && !next_worker(ps, sc, stride)) {
        it.nt = 0;
        return;
    }
    const int s = seq_of_tile(a, starts, ps.x, s_hint);
    s_hint = s;
    const int nts = starts[s + 1] - starts[s];
    const long long rb = (long long)a.Hkv * starts[s];
    const int h = (int)((ps.x - rb) / nts);
    const long long row_begin = rb + (long long)h * nts, row_end = row_begin + nts;
    const int t = (int)(ps.x - row_begin);
    const long long seg_end = min(row_end, ps.x_end);
    it.s = s;
    it.h = h;
    it.tok0 = t * kTileTok;
    it.nt = (int)(seg_end - ps.x);
    it.tok1 = min(a.seq_lens[s], (t + it.nt) * kTileTok);
    it.w = ps.w;
    it.first = ps.x == ps.x_begin || t == 0;
    it.last = true;  // an item is a whole segment
    ps.x = seg_end;
}

// Producer lane: the tile it issues next for its math warp, walked tile by
// tile through the same schedule (row s, h at tile t of nts).
struct TileWalk {
    SchedPos ps;
    int s, h, t, nts;
    int id;  // block id of the tile (read one tile ahead)
    bool live;
};

__device__ __forceinline__ void walk_locate(const DecodeArgs &a, const int32_t *starts, TileWalk &wk) {
    wk.s = seq_of_tile(a, starts, wk.ps.x, wk.s);
    wk.nts = starts[wk.s + 1] - starts[wk.s];
    const long long rel = wk.ps.x - (long long)a.Hkv * starts[wk.s];
    wk.h = (int)(rel / wk.nts);
    wk.t = (int)(rel - (long long)wk.h * wk.nts);
}

__device__ __forceinline__ int walk_block_id(const DecodeArgs &a, const TileWalk &wk) {
    return __ldg(a.block_table + (size_t)wk.s * a.max_blocks + ((wk.t * kTileTok) >> a.bs_shift));
}

// Step to the next tile (false: the math warp's schedule is done).
__device__ __forceinline__ bool walk_advance(const DecodeArgs &a, const int32_t *starts, const Sched &sc, int stride,
                                             TileWalk &wk) {
    ++wk.ps.x;
    if (wk.ps.x >= wk.ps.x_end) {
        if (!next_worker(wk.ps, sc, stride)) return false;
        walk_locate(a, starts, wk);
        return true;
    }
    if (++wk.t == wk.nts) {
        wk.t = 0;
        if (++wk.h == a.Hkv) {
            wk.h = 0;
            do {
                ++wk.s;
            } while (starts[wk.s + 1] == starts[wk.s]);  // tile x lies in a later, non-empty sequence
            wk.nts = starts[wk.s + 1] - starts[wk.s];
        }
    }
    return true;
}

// Output of a finished segment: G unnormalised rows in `scratch` ([G][d]
// fp32), row g's max / sum in lane 4g.  A row in one segment is written
// directly; otherwise the partial goes to its slot for decode_merge_kernel.
template <int G>
__device__ __forceinline__ void finish_seg(const DecodeArgs &a, const SegItem &it, const int32_t *starts,
                                           const Sched &sc, int lane, float *scratch, float m, float l, bool saw_bad) {
    const int s = it.s;
    // the row's place in the schedule: its tiles [row_begin, row_begin + nts)
    // span workers worker_of(row_begin) .. worker_of(row_begin + nts - 1)
    const int nts = starts[s + 1] - starts[s];
    const long long row_begin = (long long)a.Hkv * starts[s] + (long long)it.h * nts;
    const int r = s * a.Hkv + it.h;
    const int nsplit = (int)(worker_of(sc, row_begin + nts - 1) - worker_of(sc, row_begin)) + 1;
    const int slot = it.w + r;
    const size_t sh0 = (size_t)s * a.H + (size_t)it.h * G;
    const int gl = lane & 7;  // lanes 0..G-1: the row they report
    const float mg_l = __shfl_sync(0xffffffffu, m, 4 * gl);
    const float lg_l = __shfl_sync(0xffffffffu, l, 4 * gl);
    if (nsplit == 1) {
#pragma unroll 1
        for (int g = 0; g < G; ++g) {
            const float lg = __shfl_sync(0xffffffffu, l, 4 * g);
            const float inv = (!saw_bad && lg > 0.f) ? 1.f / lg : 0.f;
            const float4 v = *reinterpret_cast<const float4 *>(scratch + g * kD + 4 * lane);
            *reinterpret_cast<uint2 *>(a.O + (sh0 + g) * kD + 4 * lane) =
                make_uint2(pack_bf16x2(v.x * inv, v.y * inv), pack_bf16x2(v.z * inv, v.w * inv));
        }
        if (lane < G) a.LSE[sh0 + lane] = (!saw_bad && lg_l > 0.f) ? (mg_l + __log2f(lg_l)) * kLn2 : -INFINITY;
        return;
    }
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        const float lg = __shfl_sync(0xffffffffu, l, 4 * g);
        const float inv = lg > 0.f ? 1.f / lg : 0.f;
        const float4 v = *reinterpret_cast<const float4 *>(scratch + g * kD + 4 * lane);
        *reinterpret_cast<float4 *>(a.part_o + ((size_t)slot * G + g) * kD + 4 * lane) =
            make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
    }
    if (lane < G) a.part_lse[(size_t)slot * G + lane] = lg_l > 0.f ? mg_l + __log2f(lg_l) : -INFINITY;
    if (lane == 0) a.slot_bad[slot] = saw_bad ? 1 : 0;  // written for every cut segment: nothing to clear
}

template <int G>
__global__ void __launch_bounds__(kMmaThreads, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      DecodeArgs a) {
    static_assert(G == 4 || G == 8, "query group of 4 or 8");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBarOff);  // [kCons][kStages]
    uint64_t *empty = full + kCons * kStages;                       // [kCons][kStages]
    volatile int32_t *slot_bad = reinterpret_cast<int32_t *>(smem + kBadOff);
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        for (int i = 0; i < kCons * kStages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        fence_barrier_init();
    }
    pdl_wait();
    pdl_launch_dependents();  // the merge grid may be set up now; it waits for this grid's end
    const int32_t *starts = a.item_start;  // tiles before each sequence
    if (a.fused_plan) {
        // the plan, in every CTA: tiles per sequence (none for an empty or
        // invalid length) and their exclusive prefix, by a block-wide scan;
        // CTA 0 publishes it for the merge kernel
        __shared__ int warp_sum[kMmaThreads / 32];
        int32_t *st = reinterpret_cast<int32_t *>(smem + kStartsOff);
        const int n = a.num_seqs, per = (n + kMmaThreads - 1) / kMmaThreads;
        const int k0 = min(n, (int)threadIdx.x * per), k1 = min(n, k0 + per);
        auto seq_tiles = [&](int k) {
            const int L = a.seq_lens[k];
            return (L > 0 && seq_len_ok(L, a)) ? (L + kTileTok - 1) / kTileTok : 0;
        };
        int sum = 0;
        for (int k = k0; k < k1; ++k) sum += seq_tiles(k);
        int x = sum;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sum[wid] = x;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < wid; ++w) base += warp_sum[w];
        int run = base + x - sum;
        for (int k = k0; k < k1; ++k) {
            st[k] = run;
            run += seq_tiles(k);
        }
        if (threadIdx.x == kMmaThreads - 1) st[n] = base + x;
        __syncthreads();
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i <= n; i += kMmaThreads) a.item_start[i] = st[i];
        // empty and invalid sequences: O = 0, LSE = -inf (an invalid length
        // also sets its error bit); sequences spread over the CTAs
        for (int sq = blockIdx.x; sq < n; sq += gridDim.x) {
            const int L = a.seq_lens[sq];
            if (L > 0 && seq_len_ok(L, a)) continue;
            if (threadIdx.x == 0 && !seq_len_ok(L, a) && a.err) atomicOr(a.err, ATTN_DEVERR_SEQ_LEN);
            for (int e = threadIdx.x; e < a.H * (kD / 8); e += kMmaThreads)
                reinterpret_cast<uint4 *>(a.O + (size_t)sq * a.H * kD)[e] = make_uint4(0u, 0u, 0u, 0u);
            for (int hh = threadIdx.x; hh < a.H; hh += kMmaThreads) a.LSE[(size_t)sq * a.H + hh] = -INFINITY;
        }
        starts = st;
    } else if (a.num_seqs <= kMaxSmemSeqs) {
        int32_t *st = reinterpret_cast<int32_t *>(smem + kStartsOff);
        for (int i = threadIdx.x; i <= a.num_seqs; i += blockDim.x) st[i] = a.item_start[i];
        starts = st;
    }
    __syncthreads();  // barriers initialised, offsets staged
    // the schedule: T tiles in all over nw workers
    Sched sc;
    sc.T = (long long)starts[a.num_seqs] * a.Hkv;
    sc.nw = sched_nw(sc.T, a.sched_w);
    const int stride = gridDim.x * kCons;

    if (wid >= kCons) {
        // ---------------- producer warpgroup: warp kCons issues, the rest leave
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProdRegs));
        if (wid != kCons) return;
        const int c = lane;  // the math warp this lane serves
        TileWalk wk;
        wk.ps.w = blockIdx.x * kCons + c - stride;
        wk.ps.x = wk.ps.x_end = 0;
        wk.s = 0;
        wk.live = c < kCons && sc.T > 0 && next_worker(wk.ps, sc, stride);
        if (wk.live) {
            walk_locate(a, starts, wk);
            wk.id = walk_block_id(a, wk);
        }
        uint32_t gi = 0;
        uint64_t t_last = globaltimer_ns();
        bool timed_out = false;
        while (__any_sync(0xffffffffu, wk.live)) {
            bool issued = false;
            if (wk.live) {
                const int slot = gi % kStages;
                uint64_t *fb = full + c * kStages + slot;
                // a non-blocking probe: one lane's wait must not hold up the others
                if (mbar_test_wait(empty + c * kStages + slot, ((gi / kStages) & 1u) ^ 1u)) {
                    issued = true;
                    const int id = wk.id;
                    if (id < 0 || id >= a.num_blocks) {
                        // never read: the math warp skips the tile and marks the sequence
                        slot_bad[c * kStages + slot] = 1;
                        if (a.err) atomicOr(a.err, ATTN_DEVERR_BLOCK_TABLE);
                        mbar_arrive(fb);
                    } else {
                        slot_bad[c * kStages + slot] = 0;
                        const int y = ((id * a.kv_heads + wk.h / a.kv_div) << a.bs_shift) +
                                      ((wk.t * kTileTok) & (a.block_size - 1));
                        uint8_t *dst = smem + (c * kStages + slot) * kSlotBytes;
                        mbar_arrive_expect_tx(fb, kSlotBytes);
                        tma_load_2d(dst, &tmK, fb, 0, y);
                        tma_load_2d(dst + 2048, &tmK, fb, 64, y);
                        tma_load_2d(dst + kTileBytes, &tmV, fb, 0, y);
                        tma_load_2d(dst + kTileBytes + 2048, &tmV, fb, 64, y);
                    }
                    ++gi;
                    wk.live = walk_advance(a, starts, sc, stride, wk);
                    if (wk.live) wk.id = walk_block_id(a, wk);  // consumed at the next issue
                    t_last = globaltimer_ns();
                }
            }
            if (!__any_sync(0xffffffffu, issued)) {
                __nanosleep(64);  // nothing to refill: leave the issue slots to the math warps
                // bounded: a math warp that stopped consuming (its own wait ran
                // out) ends this loop after the wait limit
                if (wk.live && globaltimer_ns() - t_last > kWaitLimitNs) {
                    timed_out = true;
                    wk.live = false;
                }
            }
        }
        if (timed_out && a.err) atomicOr(a.err, ATTN_DEVERR_TIMEOUT);
        // copies still in flight land before the CTA may exit
        if (c < kCons) {
            for (uint32_t k = gi > kStages ? gi - kStages : 0; k < gi; ++k)
                mbar_wait(full + c * kStages + k % kStages, (k / kStages) & 1u, nullptr);
        }
        return;
    }

    // ---------------- math warps
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsRegs));
    const int gq = lane >> 2, tq = lane & 3;  // fragment row (query head of the group) and column pair
    uint8_t *slots = smem + (size_t)wid * kStages * kSlotBytes;
    float *scratch = reinterpret_cast<float *>(smem + kRingBytes + wid * kScratchBytes);
    uint64_t *my_full = full + wid * kStages, *my_empty = empty + wid * kStages;
    SchedPos ps;
    ps.w = blockIdx.x * kCons + wid - stride;
    ps.x = ps.x_begin = ps.x_end = 0;
    int s_hint = 0;
    uint32_t gc = 0;
    const uint32_t slots_u32 = smem_u32(slots);
    // ldmatrix row addresses of this lane inside a K or V tile: row `key` of
    // 16-byte chunk 2j + (q & 1) (j = ks & 3, plus 2048 for ks >= 4: the
    // second 64-column box), 128-byte swizzle
    uint32_t frag_off[4];
    {
        const int q = lane >> 3, key = 8 * (q >> 1) + (lane & 7);
#pragma unroll
        for (int j = 0; j < 4; ++j) frag_off[j] = sw_off(key, 2 * j + (q & 1));
    }
    for (;;) {
        SegItem cur;
        if (sc.T == 0) break;
        next_seg_item(a, starts, sc, stride, s_hint, ps, cur);
        if (cur.nt == 0) break;
        // Q fragments of the group (rows gq < G; 16-dim k-steps): a0 = dims
        // 16ks + 2tq, +1 and a2 = dims 16ks + 8 + 2tq, +1 of query head gq
        uint32_t qa0[8], qa2[8];
        {
            const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
                a.q + ((size_t)cur.s * a.H + cur.h * G + (gq < G ? gq : 0)) * kD);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qa0[ks] = gq < G ? __ldg(qrow + 8 * ks + tq) : 0u;
                qa2[ks] = gq < G ? __ldg(qrow + 8 * ks + 4 + tq) : 0u;
            }
        }
        float m = -INFINITY, l = 0.f;  // row gq: running max (log2 units) and this lane's part of the sum
        // O^T accumulators: o[mb] holds dims 16mb + gq (0, 1) and 16mb + gq + 8
        // (2, 3) of query heads 2tq (0, 2) and 2tq + 1 (1, 3)
        float o[8][4];
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) o[mb][0] = o[mb][1] = o[mb][2] = o[mb][3] = 0.f;
        bool saw_bad = false, dead = false;
        for (int t = 0; t < cur.nt; ++t, ++gc) {
            const int slot = gc % kStages;
            if (!mbar_wait(my_full + slot, (gc / kStages) & 1u, a.err)) {
                dead = true;
                break;
            }
            const int tok = cur.tok0 + t * kTileTok;
            const bool tile_ok = slot_bad[wid * kStages + slot] == 0;
            saw_bad |= !tile_ok;
            if (tile_ok) {
                const uint32_t kt = slots_u32 + slot * kSlotBytes, vt = kt + kTileBytes;
                const int valid = min(kTileTok, cur.tok1 - tok);  // live keys of the tile (>= 1)
                if (valid < kTileTok) {
                    // slots past the sequence may hold anything (NaN included) and
                    // 0 * NaN = NaN in P V: zero the dead V rows first
                    uint8_t *vrows = slots + slot * kSlotBytes + kTileBytes;
                    for (int e = lane; e < (kTileTok - valid) * 16; e += 32) {
                        const int r = valid + (e >> 4), c = e & 15;
                        *reinterpret_cast<uint4 *>(vrows + sw_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();  // before the slot's next TMA refill
                    __syncwarp();
                }
                // S = Q K^T: keys 0..7 (n-block 0) and 8..15 (n-block 1), the
                // 128 dims in two independent halves (two shorter MMA chains);
                // the asm statements keep their order, so every fragment load of
                // the tile goes out before the first MMA that needs one
                float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t vf[8][4];
                {
                    uint32_t kf[8][4];
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        ldsm_x4(kt + (ks >> 2) * 2048 + frag_off[ks & 3], kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3]);
#pragma unroll
                    for (int mb = 0; mb < 8; ++mb)
                        ldsm_x4_t(vt + (mb >> 2) * 2048 + frag_off[mb & 3], vf[mb][0], vf[mb][1], vf[mb][2], vf[mb][3]);
                    float u0[4] = {0.f, 0.f, 0.f, 0.f}, u1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        mma_bf16(s0, qa0[ks], qa2[ks], kf[ks][0], kf[ks][1]);
                        mma_bf16(s1, qa0[ks], qa2[ks], kf[ks][2], kf[ks][3]);
                        mma_bf16(u0, qa0[ks + 4], qa2[ks + 4], kf[ks + 4][0], kf[ks + 4][1]);
                        mma_bf16(u1, qa0[ks + 4], qa2[ks + 4], kf[ks + 4][2], kf[ks + 4][3]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        s0[e] += u0[e];
                        s1[e] += u1[e];
                    }
                }
                // online softmax of row gq over the tile's 16 keys (this lane:
                // keys 2tq, 2tq+1, 8+2tq, 9+2tq)
                float x[4] = {s0[0] * a.scale_log2, s0[1] * a.scale_log2, s1[0] * a.scale_log2,
                              s1[1] * a.scale_log2};
                const int kc[4] = {2 * tq, 2 * tq + 1, 8 + 2 * tq, 9 + 2 * tq};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (kc[e] >= valid) x[e] = -INFINITY;
                float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                // lazy rescaling: the reference max moves only when the tile's
                // max exceeds it by more than kLazyLog2 (always on the first
                // tile, m = -inf); otherwise the probabilities are taken
                // against the old max (at most 2^kLazyLog2) and nothing is
                // rescaled -- O, l and the max stay consistent either way
                const bool bump = mx > m + kLazyLog2;
                const float m_new = bump ? mx : m;  // finite: key 0 of every tile is live
                const float alpha = bump ? ex2_approx(m - m_new) : 1.f;
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) p[e] = ex2_approx(x[e] - m_new);
                l = l * alpha + ((p[0] + p[1]) + (p[2] + p[3]));
                m = m_new;
                if (__any_sync(0xffffffffu, bump)) {
                    // this lane's accumulators belong to query heads 2tq and 2tq + 1
                    const float al0 = __shfl_sync(0xffffffffu, alpha, 8 * tq);
                    const float al1 = __shfl_sync(0xffffffffu, alpha, 8 * tq + 4);
#pragma unroll
                    for (int mb = 0; mb < 8; ++mb) {
                        o[mb][0] *= al0;
                        o[mb][2] *= al0;
                        o[mb][1] *= al1;
                        o[mb][3] *= al1;
                    }
                }
                // P^T fragments (keys 2tq, 2tq + 1 and 8 + 2tq, 9 + 2tq of head gq)
                const uint32_t pb0 = pack_bf16x2(p[0], p[1]), pb1 = pack_bf16x2(p[2], p[3]);
                // O^T += V^T P^T: dims 16mb .. 16mb + 15 per m-block
#pragma unroll
                for (int mb = 0; mb < 8; ++mb) mma_bf16_4(o[mb], vf[mb][0], vf[mb][1], vf[mb][2], vf[mb][3], pb0, pb1);
            }
            // the P V MMAs have issued, so every fragment load of the slot has
            // completed: release it to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(my_empty + slot);
        }
        if (dead) break;
        // unnormalised O rows -> per-warp scratch, then the common finish
        // (final row, or partial + merge by the last segment)
        float lt = l + __shfl_xor_sync(0xffffffffu, l, 1);
        lt += __shfl_xor_sync(0xffffffffu, lt, 2);
        if (2 * tq < G) {
#pragma unroll
            for (int mb = 0; mb < 8; ++mb) {
                scratch[(2 * tq) * kD + 16 * mb + gq] = o[mb][0];
                scratch[(2 * tq + 1) * kD + 16 * mb + gq] = o[mb][1];
                scratch[(2 * tq) * kD + 16 * mb + gq + 8] = o[mb][2];
                scratch[(2 * tq + 1) * kD + 16 * mb + gq + 8] = o[mb][3];
            }
        }
        __syncwarp();
        finish_seg<G>(a, cur, starts, sc, lane, scratch, m, lt, saw_bad);
        __syncwarp();  // scratch reads done before the next segment writes it
    }
}

// The rows the grouped kernel left in partials, one warp per query head:
// sh = s H + hq, key/value row r = s Hkv + hq / G, the row's segments in
// slots slot0 .. slot0 + nsplit - 1 (slot0 = first worker + r).  Launched as
// a programmatic dependent of decode_mma_kernel: griddepcontrol.wait returns
// once that grid has finished and its writes are visible.  Lane j holds the
// log2-sum-exp and bad flag of partials j, j + 32, ...; the maximum and the
// weight sum are warp reductions and the weighted rows are summed in partial
// order, so the result depends only on the lengths and sizes.  The first 16
// partial rows are requested together with the log2-sum-exps.  When the
// tile kernel planned for itself, the row's place in the schedule follows
// from seq_lens alone, so it is worked out before the wait and only the
// partials are read after it.  seq_lens is an input: this grid starts only
// once every CTA of the tile kernel has passed that kernel's own dependency
// wait, so whatever wrote seq_lens before the call has completed.
__global__ void __launch_bounds__(256) decode_merge_kernel(DecodeArgs a, int G) {
    constexpr int kBatch = 16;  // partial rows in flight per lane
    const int lane = threadIdx.x & 31;
    const long long sh = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const bool have = sh < (long long)a.num_seqs * a.H;
    const int s = have ? (int)(sh / a.H) : 0, hq = have ? (int)(sh - (long long)s * a.H) : 0;
    int st0 = 0, st1 = 0, stn = 0;
    if (a.fused_plan && have) {
        // the plan's exclusive prefix at s and s + 1 and its total: tiles of
        // each sequence (none for an empty or invalid length), summed by the warp
        int before = 0, upto = 0, all = 0;
        for (int k = lane; k < a.num_seqs; k += 32) {
            const int L = __ldg(a.seq_lens + k);
            const int t = (L > 0 && seq_len_ok(L, a)) ? (L + kTileTok - 1) / kTileTok : 0;
            all += t;
            if (k < s) before += t;
            if (k <= s) upto += t;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            before += __shfl_xor_sync(0xffffffffu, before, o);
            upto += __shfl_xor_sync(0xffffffffu, upto, o);
            all += __shfl_xor_sync(0xffffffffu, all, o);
        }
        st0 = before;
        st1 = upto;
        stn = all;
    }
    pdl_wait();
    if (!have) return;
    const int h = hq / G, g = hq - h * G;
    if (!a.fused_plan) {
        const int32_t *starts = a.item_start;
        st0 = __ldcg(starts + s);
        st1 = __ldcg(starts + s + 1);
        stn = __ldcg(starts + a.num_seqs);
    }
    const int nts = st1 - st0;
    if (nts == 0) return;  // empty or invalid length: written with the plan
    Sched sc;
    sc.T = (long long)stn * a.Hkv;
    sc.nw = sched_nw(sc.T, a.sched_w);
    const long long row_begin = (long long)a.Hkv * st0 + (long long)h * nts;
    const int w0 = (int)worker_of(sc, row_begin);
    const int nsplit = (int)worker_of(sc, row_begin + nts - 1) - w0 + 1;
    if (nsplit == 1) return;  // written by its segment
    const size_t slot0 = (size_t)w0 + (size_t)s * a.Hkv + h;
    const float *plse = a.part_lse + slot0 * G + g;                                      // partial q at plse[q G]
    const float4 *po = reinterpret_cast<const float4 *>(a.part_o + (slot0 * G + g) * kD) + lane;  // po[q G d / 4]
    const int32_t *pbad = a.slot_bad + slot0;
    const float lse0 = lane < nsplit ? __ldcg(plse + (size_t)lane * G) : -INFINITY;
    int bad = lane < nsplit ? __ldcg(pbad + lane) : 0;
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
        if (u < nsplit) v[u] = __ldcg(po + (size_t)u * G * (kD / 4));
    float M = lse0;
    for (int q = 32 + lane; q < nsplit; q += 32) {
        M = fmaxf(M, __ldcg(plse + (size_t)q * G));
        bad |= __ldcg(pbad + q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (__any_sync(0xffffffffu, bad != 0)) {  // a bad block id in the row: the sequence's result is zeros
        *reinterpret_cast<uint2 *>(a.O + sh * kD + 4 * lane) = make_uint2(0u, 0u);
        if (lane == 0) a.LSE[sh] = -INFINITY;
        return;
    }
    float tot = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q0 = 0; q0 < nsplit; q0 += 32) {
        const int n = min(32, nsplit - q0);
        const float lse = q0 == 0 ? lse0 : (lane < n ? __ldcg(plse + (size_t)(q0 + lane) * G) : -INFINITY);
        const float wl = lane < n ? ex2_approx(lse - M) : 0.f;
        float part = wl;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        tot += part;
        for (int j0 = 0; j0 < n; j0 += kBatch) {
            if (q0 + j0 > 0) {
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    if (j0 + u < n) v[u] = __ldcg(po + (size_t)(q0 + j0 + u) * G * (kD / 4));
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const float w = __shfl_sync(0xffffffffu, wl, (j0 + u) & 31);
                if (j0 + u < n) {
                    acc.x = fmaf(w, v[u].x, acc.x);
                    acc.y = fmaf(w, v[u].y, acc.y);
                    acc.z = fmaf(w, v[u].z, acc.z);
                    acc.w = fmaf(w, v[u].w, acc.w);
                }
            }
        }
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    *reinterpret_cast<uint2 *>(a.O + sh * kD + 4 * lane) =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    if (lane == 0) a.LSE[sh] = tot > 0.f ? (M + __log2f(tot)) * kLn2 : -INFINITY;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
    size_t counter, item_start, done_cnt, seq_bad, slot_bad, part_lse, part_o, total;
};

// prow: partial rows (fp32 [d] each, plus a log2-sum-exp)
WsLayout ws_layout(int num_seqs, int H, size_t prow) {
    WsLayout w;
    w.counter = 0;
    w.item_start = 256;
    w.done_cnt = align_up(w.item_start + sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
    w.seq_bad = align_up(w.done_cnt + sizeof(int32_t) * (size_t)num_seqs * H, 256);
    w.slot_bad = align_up(w.seq_bad + sizeof(int32_t) * (size_t)num_seqs, 256);
    w.part_lse = align_up(w.slot_bad + sizeof(int32_t) * (prow / 4 + 1), 256);  // slots hold >= 4 rows
    w.part_o = align_up(w.part_lse + sizeof(float) * prow, 256);
    w.total = align_up(w.part_o + sizeof(float) * prow * kD, 256);
    return w;
}

// Partial rows for these sizes: [num_seqs, H, max_splits] for the split
// kernel; groups of 4 or more may run the scheduled kernel, whose slots hold
// at most (workers + num_seqs * H / G) x G rows (G <= 8 per slot).
size_t partial_rows(int num_seqs, int H, int Hkv, int max_splits) {
    const size_t split_rows = (size_t)num_seqs * H * (size_t)(max_splits < 1 ? 1 : max_splits);
    if (H / Hkv < 4) return split_rows;
    const size_t sched_rows = (size_t)kMaxWorkers * 8 + (size_t)num_seqs * H;
    return split_rows > sched_rows ? split_rows : sched_rows;
}

}  // namespace

int decode_split_tokens(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size) {
    (void)d;
    const long long max_len = (long long)max_blocks * block_size;
    const long long work = (long long)num_seqs * H * max_len;
    // (the grouping does not change the split: half-length splits for groups
    // of 4 and 8, which would double the items, measured slower -- more
    // partials, fences and merges than the tail they save)
    (void)Hkv;
    long long split = 256;
    // larger splits for large problems (bounded workspace), at most 64 blocks
    // per split (the kernel keeps a split's block ids in two registers per lane)
    while (split < max_len && work / split > 65536 && split * 2 <= 64LL * block_size) split <<= 1;
    return (int)split;
}

int decode_max_splits(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size) {
    const long long max_len = (long long)max_blocks * block_size;
    const int split = decode_split_tokens(num_seqs, H, Hkv, d, max_blocks, block_size);
    return (int)((max_len + split - 1) / split);
}

size_t decode_workspace_bytes(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size) {
    const int ms = decode_max_splits(num_seqs, H, Hkv, d, max_blocks, block_size);
    return ws_layout(num_seqs, H, partial_rows(num_seqs, H, Hkv, ms)).total;
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

template <int G>
attn_status launch_mma(const DecodeArgs &a, const DecodeLaunch &p, int dev, int sms, cudaStream_t stream) {
    static bool attr_set[64] = {false};
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(decode_mma_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMmaSmem) !=
            cudaSuccess)
            return ATTN_ECUDA;
        attr_set[dev] = true;
    }
    const long long rows = (long long)p.num_blocks * a.kv_heads * p.block_size;
    CUtensorMap tk, tv;
    if (!make_tensor_map_2d_bf16(&tk, p.k_cache, kD, rows, kD, kTileTok) ||
        !make_tensor_map_2d_bf16(&tv, p.v_cache, kD, rows, kD, kTileTok))
        return ATTN_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(kMmaThreads);
    cfg.dynamicSmemBytes = kMmaSmem;
    // the schedule's width: every math warp of the launch (the workspace holds
    // the slots of at most kMaxWorkers)
    DecodeArgs am = a;
    am.sched_w = sms * kCons < kMaxWorkers ? sms * kCons : kMaxWorkers;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_mma_kernel<G>, tk, tv, am) != cudaSuccess) return ATTN_ECUDA;
    // the rows left in partials, merged by a programmatic dependent
    const long long rows_q = (long long)a.num_seqs * a.H;
    cudaLaunchConfig_t mcfg = cfg;
    mcfg.gridDim = dim3((unsigned)((rows_q + 7) / 8));
    mcfg.blockDim = dim3(256);
    mcfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&mcfg, decode_merge_kernel, am, G) == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
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
    a.kv_heads = p.Hkv;
    a.kv_div = 1;
    a.num_blocks = p.num_blocks;
    a.max_blocks = p.max_blocks;
    a.block_size = p.block_size;
    a.bs_shift = p.block_size == 32 ? 5 : 4;
    if (G % 8 == 0 && G > 8) {
        // larger groups (multi-query attention): each cache head serves G / 8
        // virtual key/value heads of 8 query heads, adjacent in the schedule,
        // so a cache head's tiles are re-read from L2
        a.kv_div = G / 8;
        a.Hkv = p.H / 8;
    }
    // the scheduled tensor-core kernel for groups of 4 and more, unless a TMA
    // row coordinate (32-bit) or the tile count would overflow
    const long long kv_rows = (long long)p.num_blocks * p.Hkv * p.block_size;
    const long long max_tiles = ((long long)p.max_blocks * p.block_size + kTileTok - 1) / kTileTok;
    const bool sched = G >= 4 && kv_rows <= 0x7fffffffLL && (long long)p.num_seqs * max_tiles <= 0x3fffffffLL;
    if (G >= 4 && !sched && a.kv_div > 1) return ATTN_EUNSUPPORTED;
    const int ms = decode_max_splits(p.num_seqs, p.H, p.Hkv, p.d, p.max_blocks, p.block_size);
    // the plan's per-sequence counts: 16-token tiles for the schedule, splits otherwise
    a.split_tokens = sched ? kTileTok : decode_split_tokens(p.num_seqs, p.H, p.Hkv, p.d, p.max_blocks, p.block_size);
    a.max_splits = ms < 1 ? 1 : ms;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    const WsLayout w = ws_layout(p.num_seqs, p.H, partial_rows(p.num_seqs, p.H, p.Hkv, ms));
    uint8_t *ws = static_cast<uint8_t *>(p.workspace);
    a.counter = reinterpret_cast<int32_t *>(ws + w.counter);
    a.item_start = reinterpret_cast<int32_t *>(ws + w.item_start);
    a.done_cnt = reinterpret_cast<int32_t *>(ws + w.done_cnt);
    a.seq_bad = reinterpret_cast<int32_t *>(ws + w.seq_bad);
    a.slot_bad = reinterpret_cast<int32_t *>(ws + w.slot_bad);
    a.part_lse = reinterpret_cast<float *>(ws + w.part_lse);
    a.part_o = reinterpret_cast<float *>(ws + w.part_o);

    // the grouped kernel plans in every CTA when the offsets fit in shared memory
    a.fused_plan = sched && p.num_seqs <= kMaxSmemSeqs ? 1 : 0;
    a.sched_w = 0;  // set by launch_mma
    if (!a.fused_plan) {
        decode_plan_kernel<<<1, 1024, 0, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ECUDA;
    }
    if (sched) return G == 4 ? launch_mma<4>(a, p, dev, sm_count[dev], stream)
                             : launch_mma<8>(a, p, dev, sm_count[dev], stream);
    switch (G) {
        case 1: return launch_split<1>(a, dev, sm_count[dev], stream);
        case 2: return launch_split<2>(a, dev, sm_count[dev], stream);
        case 4: return launch_split<4>(a, dev, sm_count[dev], stream);
        case 8: return launch_split<8>(a, dev, sm_count[dev], stream);
    }
    return ATTN_EUNSUPPORTED;
}

}  // namespace osp
