// cow_plan.cu -- host half of copy-on-write for the paged KV cache.
//
// Method: "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解",
// section 三 内存共享机制: blocks shared by several sequences (a common
// prefix, parallel samples) carry a reference count; before a sequence
// writes into a shared block, the block is copied to a free one, the
// writer's block-table entry is pointed at the copy and the counts are
// adjusted, so the other sharers keep the old contents.  The copy itself is
// paged_block_copy's kernel; this file decides which copies a batch of
// pending writes needs and edits the caller's host-side tables.  It runs on
// the CPU, touches no device memory and allocates nothing.
#include <cstdint>

#include "../../include/attn.h"

namespace {

// Undo copy k of a batch: the write whose table entry now holds dst_out[k]
// (free blocks are unique, so exactly one entry does) goes back to
// src_out[k], the counts are restored and the block returns to the free list.
void undo_copy(int32_t *block_table, int max_blocks_per_seq, int32_t *ref_counts, int32_t *free_list,
               int32_t *free_count, const int32_t *write_seqs, const int32_t *write_blocks, int num_writes,
               int32_t src, int32_t dst) {
    for (int i = num_writes - 1; i >= 0; --i) {
        int32_t &e = block_table[(size_t)write_seqs[i] * max_blocks_per_seq + write_blocks[i]];
        if (e == dst) {
            e = src;
            break;
        }
    }
    ref_counts[src] += 1;
    ref_counts[dst] = 0;
    free_list[(*free_count)++] = dst;
}

}  // namespace

extern "C" ATTN_API attn_status paged_cow_plan(int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                                               int32_t *ref_counts, int num_blocks, int32_t *free_list,
                                               int32_t *free_count, const int32_t *write_seqs,
                                               const int32_t *write_blocks, int num_writes, int32_t *src_out,
                                               int32_t *dst_out, int32_t *num_copies) {
    if (num_seqs < 0 || max_blocks_per_seq < 1 || num_blocks < 1 || num_writes < 0) return ATTN_EINVAL;
    if (!num_copies || !free_count || *free_count < 0) return ATTN_EINVAL;
    *num_copies = 0;
    if (num_writes == 0) return ATTN_OK;
    if (!block_table || !ref_counts || !write_seqs || !write_blocks || !src_out || !dst_out) return ATTN_EINVAL;
    if (*free_count > 0 && !free_list) return ATTN_EINVAL;
    // every write names a table entry that holds a referenced block
    for (int i = 0; i < num_writes; ++i) {
        const int32_t s = write_seqs[i], lb = write_blocks[i];
        if (s < 0 || s >= num_seqs || lb < 0 || lb >= max_blocks_per_seq) return ATTN_EINVAL;
        const int32_t p = block_table[(size_t)s * max_blocks_per_seq + lb];
        if (p < 0 || p >= num_blocks || ref_counts[p] < 1) return ATTN_EINVAL;
    }
    // the writes in order; a failure part way undoes the copies made so far,
    // newest first, so the caller's arrays are as they were
    int32_t n = 0;
    attn_status st = ATTN_OK;
    for (int i = 0; i < num_writes; ++i) {
        int32_t &e = block_table[(size_t)write_seqs[i] * max_blocks_per_seq + write_blocks[i]];
        const int32_t p = e;
        if (ref_counts[p] == 1) continue;  // the writer owns the block: it writes in place
        if (*free_count == 0) {
            st = ATTN_ENOBLOCKS;
            break;
        }
        const int32_t f = free_list[*free_count - 1];
        if (f < 0 || f >= num_blocks || ref_counts[f] != 0) {
            st = ATTN_EINVAL;  // a "free" block that is out of range or still referenced
            break;
        }
        --*free_count;
        ref_counts[p] -= 1;
        ref_counts[f] = 1;
        e = f;
        src_out[n] = p;
        dst_out[n] = f;
        ++n;
    }
    if (st != ATTN_OK) {
        for (int k = n - 1; k >= 0; --k)
            undo_copy(block_table, max_blocks_per_seq, ref_counts, free_list, free_count, write_seqs, write_blocks,
                      num_writes, src_out[k], dst_out[k]);
        return st;
    }
    *num_copies = n;
    return ATTN_OK;
}
