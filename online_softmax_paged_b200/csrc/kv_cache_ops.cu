// kv_cache_ops.cu -- the two KV-cache writes around paged decode: appending
// new tokens' keys/values into block-table-addressed slots, and the block copy
// of copy-on-write.
//
// Method (pages): "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
// section 三 核心原理 -- a new token's K/V goes into its sequence's current
// block (the block table maps the logical block to a physical one), and
// sequences sharing a prompt point at the same physical blocks until one
// writes, when the block is first copied (写时复制).  "第 2 章核心模块：
// FlashAttention-2 与 PagedAttention 实现解析" section 2.2 (block table lookup).
//
// Both are pure data movement (HBM-bound): 16-byte vector loads and stores,
// each thread issuing all its loads of a round before its first store (4
// per thread per token for the append, 8 for the copy); one CTA per token
// (append); the copy runs grid-stride over 32 KiB chunks of (pair, K|V) so
// the last wave is a fraction of a chunk, not of a block.
// Out-of-range ids are skipped on the device and reported through err_flag,
// never dereferenced.
#include <cuda_runtime.h>

#include <cstdint>

#include "launch.h"
#include "ptx.cuh"

namespace osp {
namespace {

struct AppendArgs {
    const uint8_t *k_new, *v_new;
    const int32_t *seq_ids, *positions, *block_table;
    uint8_t *k_cache, *v_cache;
    int32_t *err;
    int num_seqs, max_blocks, num_blocks, H, block_size;
    int row_bytes;  // d * element size (a multiple of 16)
};

constexpr int kAppendUnroll = 4;

__global__ void __launch_bounds__(256) kv_append_kernel(AppendArgs a) {
    __shared__ long long dst_row;  // element row index of (phys, h = 0, slot), or -1
    const int t = blockIdx.x;
    if (threadIdx.x == 0) {
        const int s = a.seq_ids[t], pos = a.positions[t];
        long long r = -1;
        if (s < 0 || s >= a.num_seqs || pos < 0 || (long long)pos >= (long long)a.max_blocks * a.block_size) {
            if (a.err) atomicOr(a.err, ATTN_DEVERR_INDEX);
        } else {
            const int phys = a.block_table[(size_t)s * a.max_blocks + pos / a.block_size];
            if (phys < 0 || phys >= a.num_blocks) {
                if (a.err) atomicOr(a.err, ATTN_DEVERR_BLOCK_TABLE);
            } else {
                r = (long long)phys * a.H * a.block_size + pos % a.block_size;
            }
        }
        dst_row = r;
    }
    __syncthreads();
    const long long r0 = dst_row;
    if (r0 < 0) return;
    const int cpr = a.row_bytes / 16;  // 16-byte chunks per head row
    const int per = a.H * cpr;
    // kAppendUnroll chunks per thread per round, all loads issued before the
    // first store (a token is 2 H d-element rows: 16 KiB at H = 32, d = 128,
    // one round of 256 threads)
    for (int c0 = threadIdx.x; c0 < 2 * per; c0 += kAppendUnroll * blockDim.x) {
        uint4 x[kAppendUnroll];
        uint8_t *dst[kAppendUnroll];
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u) {
            const int c = c0 + u * blockDim.x;
            dst[u] = nullptr;
            if (c < 2 * per) {
                const int which = c >= per;
                const int rem = c - which * per;
                const int h = rem / cpr, q = rem - h * cpr;
                const uint8_t *src = (which ? a.v_new : a.k_new) + ((size_t)t * a.H + h) * a.row_bytes + 16 * q;
                dst[u] = (which ? a.v_cache : a.k_cache) + ((size_t)r0 + (size_t)h * a.block_size) * a.row_bytes +
                         16 * q;
                x[u] = __ldg(reinterpret_cast<const uint4 *>(src));
            }
        }
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u)
            if (dst[u]) *reinterpret_cast<uint4 *>(dst[u]) = x[u];
    }
}

struct CopyArgs {
    uint8_t *k_cache, *v_cache;
    const int32_t *src, *dst;
    int32_t *err;
    int num_blocks, num_pairs;
    long long block_bytes;  // H * block_size * d * element size (a multiple of 16)
    int chunks;             // 32 KiB chunks per block (the last one may be short)
};

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 8;                                 // 16-byte words in flight per thread
constexpr int kChunkBytes = kCopyThreads * kCopyUnroll * 16;  // 32 KiB

// Work unit w: pair w / (2 chunks), K (0) or V (1), chunk; each thread moves
// kCopyUnroll x 16 bytes with all loads issued before the first store.
__global__ void __launch_bounds__(kCopyThreads) block_copy_kernel(CopyArgs a) {
    const long long units = (long long)a.num_pairs * 2 * a.chunks;
    for (long long w = blockIdx.x; w < units; w += gridDim.x) {
        const int i = (int)(w / (2 * a.chunks));
        const int rem = (int)(w - (long long)i * 2 * a.chunks);
        const int which = rem / a.chunks, c = rem - which * a.chunks;
        const int s = a.src[i], d = a.dst[i];
        if (s < 0 || s >= a.num_blocks || d < 0 || d >= a.num_blocks) {
            if (threadIdx.x == 0 && which == 0 && c == 0 && a.err) atomicOr(a.err, ATTN_DEVERR_BLOCK_TABLE);
            continue;
        }
        uint8_t *base = which ? a.v_cache : a.k_cache;
        const long long off = (long long)c * kChunkBytes;
        const long long n = min((long long)kChunkBytes, a.block_bytes - off) / 16;  // 16-byte words of the chunk
        const uint4 *from = reinterpret_cast<const uint4 *>(base + (size_t)s * a.block_bytes + off);
        uint4 *to = reinterpret_cast<uint4 *>(base + (size_t)d * a.block_bytes + off);
        const int t = threadIdx.x;
        if (n == kChunkBytes / 16) {
            uint4 x[kCopyUnroll];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) x[u] = from[t + u * kCopyThreads];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) to[t + u * kCopyThreads] = x[u];
        } else {
            for (long long k = t; k < n; k += kCopyThreads) to[k] = from[k];
        }
    }
}

}  // namespace

attn_status launch_kv_append(const AppendLaunch &p, cudaStream_t stream) {
    AppendArgs a;
    a.k_new = static_cast<const uint8_t *>(p.k_new);
    a.v_new = static_cast<const uint8_t *>(p.v_new);
    a.seq_ids = p.seq_ids;
    a.positions = p.positions;
    a.block_table = p.block_table;
    a.k_cache = static_cast<uint8_t *>(p.k_cache);
    a.v_cache = static_cast<uint8_t *>(p.v_cache);
    a.err = p.err_flag;
    a.num_seqs = p.num_seqs;
    a.max_blocks = p.max_blocks;
    a.num_blocks = p.num_blocks;
    a.H = p.H;
    a.block_size = p.block_size;
    a.row_bytes = p.d * p.elem_bytes;
    kv_append_kernel<<<p.num_tokens, 256, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

attn_status launch_block_copy(const CopyLaunch &p, cudaStream_t stream) {
    CopyArgs a;
    a.k_cache = static_cast<uint8_t *>(p.k_cache);
    a.v_cache = static_cast<uint8_t *>(p.v_cache);
    a.src = p.src_blocks;
    a.dst = p.dst_blocks;
    a.err = p.err_flag;
    a.num_blocks = p.num_blocks;
    a.block_bytes = (long long)p.H * p.block_size * p.d * p.elem_bytes;
    a.num_pairs = p.num_pairs;
    a.chunks = (int)((a.block_bytes + kChunkBytes - 1) / kChunkBytes);
    static int sm_count[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ATTN_ECUDA;
    if (sm_count[dev] == 0 &&
        cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return ATTN_ECUDA;
    const long long units = (long long)p.num_pairs * 2 * a.chunks;
    const long long slots = 8LL * sm_count[dev];  // 8 resident 256-thread CTAs per SM
    const int grid = (int)(units < slots ? units : slots);
    if (grid == 0) return ATTN_OK;
    block_copy_kernel<<<grid, kCopyThreads, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ECUDA;
}

}  // namespace osp
