/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention forward library.
 *
 * Two entry points compute O = softmax(scale * Q K^T) V with online softmax
 * (a running max m and sum l per query row, the O accumulator rescaled as new
 * key tiles arrive) and emit the per-row logsumexp:
 *
 *   attn_fwd           dense prefill, causal or not, [B, H, N, d] tensors.
 *   paged_attn_decode  one query token per sequence; keys and values are read
 *                      from a paged KV cache through a per-sequence block
 *                      table of fixed-size blocks.
 *
 * Sources:
 *   "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解",
 *     section 一 (standard self-attention; formula image lost, read as
 *     softmax(Q K^T / sqrt(d)) V), section 二 核心原理 (tiling, safe softmax,
 *     stored statistics), section 二 FlashAttention-2 改进 (keep only the
 *     logsumexp), section 三 核心原理 (blocks of 16 or 32 tokens, block table
 *     from contiguous logical to non-contiguous physical blocks).
 *   "第 2 章核心模块：FlashAttention-2 与 PagedAttention 实现解析",
 *     section 2.1 (incremental normalisation), section 2.2 (paged loop).
 *   "Transformer内存优化：从Flash Attention到Page Attention", section 1.1
 *     (layout [batch, heads, seq_len, dim]).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory and keeps no pointer after return.
 *     (paged_cow_plan, the host half of copy-on-write, is the exception: it
 *     edits HOST arrays and makes no device call.)
 *   - Calls are asynchronous on `stream` (0 = legacy default stream); nothing
 *     synchronises the host.  Outputs are valid once the stream reaches the
 *     launch.
 *   - Tensors are contiguous, row-major, in the shapes stated, and 16-byte
 *     aligned.  Inputs are read-only; outputs are written completely.
 *   - Host-side argument checks run before any launch and return
 *     ATTN_EINVAL or ATTN_EUNSUPPORTED with nothing launched.  A failed launch
 *     returns ATTN_ECUDA.  Problems only the device can see (a block-table
 *     entry out of range, a sequence length out of range, a pipeline wait
 *     that exceeded its iteration limit) are OR-ed into `*err_flag` (a
 *     caller-zeroed device int32, may be NULL) as ATTN_DEVERR_* bits; the
 *     kernels never trap.  attn_read_error() turns the flag into a status.
 *   - LSE is the natural logarithm of sum_j exp(scale * q . k_j), fp32.
 */
#ifndef ONLINE_SOFTMAX_PAGED_ATTN_H
#define ONLINE_SOFTMAX_PAGED_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *attn_stream_t; /* same type as cudaStream_t */

typedef enum {
    ATTN_OK = 0,
    ATTN_EINVAL = 1,       /* bad pointer, size, alignment or shape */
    ATTN_EUNSUPPORTED = 2, /* valid but not implemented (head dim, dtype) */
    ATTN_ECUDA = 3,        /* a CUDA runtime / driver call failed */
    ATTN_EDEVICE = 4,      /* the device reported a problem via err_flag */
    ATTN_ENOBLOCKS = 5     /* paged_cow_plan: the free list ran out */
} attn_status;

typedef enum { ATTN_F32 = 0, ATTN_BF16 = 1 } attn_dtype;

/* Bits the kernels OR into *err_flag. */
#define ATTN_DEVERR_BLOCK_TABLE 1 /* block_table entry outside [0, num_blocks) */
#define ATTN_DEVERR_SEQ_LEN 2     /* seq_len < 0 or > max_blocks_per_seq * block_size */
#define ATTN_DEVERR_TIMEOUT 4     /* a pipeline wait exceeded its iteration limit */
#define ATTN_DEVERR_INDEX 8       /* a token's sequence id or position out of range */

/*
 * Dense attention forward (prefill).
 *
 * Q, K, V, O : [B, H, N, d] of `dt` (ATTN_BF16 or ATTN_F32).
 * LSE        : [B, H, N] fp32.
 * causal     : nonzero -> query row i sees keys 0..i (square, Nq = Nk = N).
 * scale      : multiplies q . k (normally 1/sqrt(d)); must be finite and > 0.
 * Supported  : d in {64, 128}; N >= 1; B * H >= 1.  bf16 runs on the
 *              tcgen05 tensor cores with fp32 accumulation (P is rounded to
 *              bf16 before the P V product); fp32 runs on CUDA cores in fp32.
 * err_flag   : optional device int32, see the conventions above.
 * Result     : O_i = sum_j softmax_j(scale q_i . k_j) v_j in `dt`,
 *              LSE_i = ln sum_j exp(scale q_i . k_j).
 */
ATTN_API attn_status attn_fwd(const void *Q, const void *K, const void *V, void *O, float *LSE,
                     int B, int H, int N, int d, int causal, float scale,
                     attn_dtype dt, int32_t *err_flag, attn_stream_t stream);

/*
 * Bytes of device workspace paged_attn_decode needs for these sizes (split-KV
 * partial outputs and their logsumexps).  Returns 0 for invalid sizes.
 */
ATTN_API size_t paged_attn_decode_workspace_size(int num_seqs, int H, int d, int max_blocks_per_seq,
                                        int block_size);

/*
 * Bytes of device workspace paged_attn_decode_gqa needs (H_q query heads over
 * H_kv key/value heads).  Returns 0 for invalid sizes (H_q not a multiple of
 * H_kv, or as paged_attn_decode_workspace_size).  At least
 * paged_attn_decode_workspace_size(num_seqs, H_q, ...): groups of 4 and more
 * also need room for the partial rows of their balanced schedule (at most
 * 1480 x 8 + num_seqs x H_q rows of d + 1 floats), which is more for few
 * short sequences.  Callers of paged_attn_decode_gqa size with this one.
 */
ATTN_API size_t paged_attn_decode_gqa_workspace_size(int num_seqs, int H_q, int H_kv, int d,
                                                     int max_blocks_per_seq, int block_size);

/*
 * Tokens per split-KV chunk the decode uses for these sizes (a function of
 * the sizes only, never of the data; exposed for tests and tooling).
 */
ATTN_API int paged_attn_decode_split_tokens(int num_seqs, int H, int d, int max_blocks_per_seq,
                                   int block_size);

/*
 * Paged decode: one query token per sequence against its cached keys/values.
 *
 * q            : [num_seqs, H, d] bf16.
 * k_cache,
 * v_cache      : [num_blocks, H, block_size, d] bf16 (a block holds
 *                block_size consecutive tokens of one sequence, all heads).
 * block_table  : int32 [num_seqs, max_blocks_per_seq]; entry [s][lb] is the
 *                physical block holding logical block lb (tokens
 *                lb*block_size ..) of sequence s.  Entries past a sequence's
 *                last block are never read.  Several sequences may name the
 *                same physical block (shared prefix, read-only).
 * seq_lens     : int32 [num_seqs]; the number of cached tokens the query
 *                attends to (its own token included if it was written).
 * O            : [num_seqs, H, d] bf16.   LSE : [num_seqs, H] fp32.
 * workspace    : device buffer of at least
 *                paged_attn_decode_workspace_size(...) bytes, 16-byte
 *                aligned, contents ignored on entry and clobbered.
 * Supported    : bf16; d = 128; block_size in {16, 32}.
 * Device checks: a block-table entry outside [0, num_blocks) or a seq_len
 *                outside [0, max_blocks_per_seq * block_size] sets the
 *                matching ATTN_DEVERR_* bit; that sequence's O is written as
 *                0 and its LSE as -inf, and no out-of-range address is read.
 * seq_len == 0 : O = 0, LSE = -inf (no error).
 * Determinism  : the split plan and every reduction order depend only on the
 *                sizes and the sequence lengths, never on the physical block
 *                ids, so moving blocks to other physical ids (with a matching
 *                table) gives bit-identical results.
 */
ATTN_API attn_status paged_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_table, const int32_t *seq_lens, int block_size,
                              void *O, float *LSE,
                              int num_seqs, int H, int d, int num_blocks, int max_blocks_per_seq,
                              float scale, attn_dtype dt, void *workspace, size_t workspace_bytes,
                              int32_t *err_flag, attn_stream_t stream);

/*
 * Grouped-query paged decode: H_q query heads share H_kv key/value heads,
 * query head h reading key/value head h / (H_q / H_kv) (multi-query attention
 * is H_kv = 1).  The pages describe multi-head attention only; this is the
 * same decode with the group mapping.
 *
 * q, O         : [num_seqs, H_q, d] bf16;   LSE : [num_seqs, H_q] fp32.
 * k_cache,
 * v_cache      : [num_blocks, H_kv, block_size, d] bf16.
 * workspace    : paged_attn_decode_gqa_workspace_size(num_seqs, H_q, H_kv, d, ...) bytes.
 * Supported    : H_q / H_kv in {1, 2, 4} or a multiple of 8 (multi-query
 *                attention included: groups above 8 run as groups of 8
 *                sharing a key/value head, whose tiles are then read from
 *                L2 after the first); otherwise as paged_attn_decode
 *                (whose behaviour, checks and determinism apply unchanged;
 *                paged_attn_decode is this call with H_kv = H_q).
 * Schedule     : groups of 4 and more cut the (sequence, key/value head)
 *                rows, laid end to end, into equal runs of 16-token tiles,
 *                one per worker (1184 workers, runs of at least 128 tokens),
 *                so a call's split plan depends on every sequence's length;
 *                rows cut into several runs are merged by a second kernel
 *                on the same stream.
 *                Groups above 8 return ATTN_EUNSUPPORTED when
 *                num_blocks * H_kv * block_size exceeds 2^31 - 1 rows or
 *                num_seqs * ceil(max_blocks_per_seq * block_size / 16)
 *                exceeds 2^30 - 1 (groups of 4 and 8 then run the
 *                split-KV kernel instead).
 */
ATTN_API attn_status paged_attn_decode_gqa(const void *q, const void *k_cache, const void *v_cache,
                                           const int32_t *block_table, const int32_t *seq_lens, int block_size,
                                           void *O, float *LSE, int num_seqs, int H_q, int H_kv, int d,
                                           int num_blocks, int max_blocks_per_seq, float scale, attn_dtype dt,
                                           void *workspace, size_t workspace_bytes, int32_t *err_flag,
                                           attn_stream_t stream);

/*
 * FP8 prefill, step 1: block quantisation of Q or K to e4m3
 * ("一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解" §二
 * "FlashAttention-3改进": the GEMMs run on FP8 tensor cores; block
 * quantisation and incoherent processing limit the accuracy lost).
 *
 * x      : bf16 [BH, N, d] (device), d = 128.
 * codes  : e4m3 [BH, N, d] (device, one byte per element, caller-owned).
 * scales : fp32 [BH, ceil(N / 128)] (device): one dequantisation scale per
 *          block of 128 rows of one head.
 * signs  : null, or d int8 values of +1 / -1 (device): incoherent processing,
 *          each row is multiplied by diag(signs) and the Sylvester Hadamard
 *          matrix before quantisation.  Give Q and K the same signs: the
 *          1/sqrt(d) of the rotation is folded into the scales, so the
 *          dequantised operands keep Q K^T.
 * Per block: amax = max |y| (y the rotated or plain rows, fp32);
 * code = e4m3(y * fp32(448 / amax)) rounded to nearest even, saturating;
 * scale = amax / 448 (/ sqrt(d) with rotation); an all-zero block has
 * scale 1 and zero codes.
 * Errors: ATTN_EUNSUPPORTED for d != 128; ATTN_EINVAL for null or unaligned
 * pointers (x, codes 16-byte; scales 4-byte).  BH = 0 or N = 0: no-op.
 */
ATTN_API attn_status attn_quantize_fp8(const void *x, void *codes, float *scales, int BH, int N, int d,
                                       const int8_t *signs, attn_stream_t stream);

/*
 * FP8 prefill, step 2: attn_fwd with e4m3 Q and K (from attn_quantize_fp8)
 * and bf16 V.  S = (Q8 * q_scale)(K8 * k_scale)^T is computed on tcgen05
 * tensor cores (kind::f8f6f4, fp32 accumulation); the per-block scales
 * fold into the softmax scale, so the online softmax, P.V (bf16) and the
 * outputs are those of attn_fwd.  O bf16 [B, H, N, d], LSE fp32 [B, H, N];
 * d = 128; causal as attn_fwd.
 * Errors: as attn_fwd (q8, k8, V, O 16-byte aligned; scales and LSE 4-byte).
 */
ATTN_API attn_status attn_fwd_fp8(const void *q8, const float *q_scale, const void *k8, const float *k_scale,
                                  const void *V, void *O, float *LSE, int B, int H, int N, int d, int causal,
                                  float scale, int32_t *err_flag, attn_stream_t stream);

/*
 * Multi-token paged prefill (chunked prefill / prefix reuse): several new
 * query tokens per sequence attend causally to that sequence's paged cache,
 * which already holds their own keys and values ("第 2 章核心模块：
 * FlashAttention-2 与 PagedAttention 实现解析" section 2.2 runs the paged loop
 * for each query position; section 2.3 pairs PagedAttention's storage with
 * FlashAttention's tiled computation).
 *
 * q, O         : [total_q, H_q, d] bf16, the new tokens of all sequences
 *                packed: sequence s owns rows cu_q[s] .. cu_q[s+1]-1.
 * LSE          : [total_q, H_q] fp32.
 * cu_q         : int32 [num_seqs + 1], cu_q[0] = 0, non-decreasing.
 * seq_lens     : int32 [num_seqs], keys cached for each sequence including
 *                its n_s = cu_q[s+1] - cu_q[s] new tokens; new token i of
 *                sequence s is at position seq_lens[s] - n_s + i and sees
 *                keys 0 .. that position.
 * block_table,
 * caches       : as for paged_attn_decode_gqa (H_kv key/value heads; query
 *                head h reads key/value head h / (H_q / H_kv)).
 * max_q_per_seq: an upper bound of n_s (host value; sizes the work grid).
 * Supported    : bf16; d in {64, 128}; block_size in {16, 32}.  Runs on the
 *                tcgen05 prefill kernel, one TMA box per cache block.
 * Device checks: a table entry outside [0, num_blocks) sets
 *                ATTN_DEVERR_BLOCK_TABLE (block 0 is read in its place and the
 *                sequence's rows are not meaningful); cu_q entries outside
 *                [0, total_q] or decreasing set ATTN_DEVERR_INDEX; a sequence
 *                with n_s > seq_lens[s] or seq_lens[s] > max_blocks_per_seq *
 *                block_size sets ATTN_DEVERR_SEQ_LEN.  The rows of a sequence
 *                flagged by either of the last two are not written.
 * Cache slots past seq_lens[s] may hold any bits (NaN included): they take
 *                no part in the product.
 */
ATTN_API attn_status paged_attn_prefill(const void *q, const void *k_cache, const void *v_cache,
                                        const int32_t *block_table, const int32_t *seq_lens, const int32_t *cu_q,
                                        int block_size, void *O, float *LSE, int num_seqs, int total_q,
                                        int max_q_per_seq, int H_q, int H_kv, int d, int num_blocks,
                                        int max_blocks_per_seq, float scale, attn_dtype dt, int32_t *err_flag,
                                        attn_stream_t stream);

/*
 * Paged decode without a workspace argument, for callers that cannot
 * allocate device memory (code running where cudaMalloc is not permitted or
 * not wanted, e.g. inside an allocator or pool callback, in a process whose
 * device memory is fixed up front, or a plain C program with no framework to
 * borrow memory from).  The pages have no counterpart: this is a deployment
 * convenience, not part of the method.
 *
 * Arguments, layouts, results and device checks are those of
 * paged_attn_decode.  The split-KV scratch is a fixed array of
 * ATTN_NOALLOC_SCRATCH_BYTES compiled into the library, reserved on every GPU
 * that loads the library for the life of the process; the call itself
 * allocates nothing.
 *   - Sizes whose workspace (paged_attn_decode_workspace_size) exceeds
 *     ATTN_NOALLOC_SCRATCH_BYTES return ATTN_EUNSUPPORTED, nothing launched.
 *   - Every call on a device shares the one scratch array: calls whose
 *     kernels can overlap on the GPU (streams without ordering between them)
 *     race and give wrong results.  Calls on one stream are safe.
 *   - The scratch keeps the previous call's contents; whatever must start at
 *     zero (the work counter, the completion counts, the bad-block marks) is
 *     cleared by the call itself.
 *   - The scratch used is the current device's: make the device that holds
 *     the tensors current (cudaSetDevice) before the call.
 *   - The first call made while a device is current looks up the scratch
 *     address with a runtime call; make that first call before any stream
 *     capture starts.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
ATTN_API attn_status paged_attn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                      const int32_t *block_table, const int32_t *seq_lens, int block_size,
                                      void *O, float *LSE,
                                      int num_seqs, int H, int d, int num_blocks, int max_blocks_per_seq,
                                      float scale, attn_dtype dt, int32_t *err_flag, attn_stream_t stream);

/*
 * Append new tokens' keys and values to the paged cache: the write that
 * precedes decode ("一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解",
 * section 三 核心原理: a new token goes into the sequence's current block,
 * found through its block table; allocating that block is the caller's job).
 *
 * k_new, v_new : [num_tokens, H, d] of `dt`; token t belongs to sequence
 *                seq_ids[t] at position positions[t] (int32 arrays).
 * block_table  : int32 [num_seqs, max_blocks_per_seq], as for decode.
 * k_cache,
 * v_cache      : [num_blocks, H, block_size, d] of `dt`, written in place:
 *                cache[block_table[s][pos / block_size], h, pos % block_size, :]
 *                = new[t, h, :] for every head h.
 * Supported    : ATTN_BF16 or ATTN_F32; d in {64, 128}; block_size in {16, 32}.
 * Device checks: a sequence id or position out of range sets
 *                ATTN_DEVERR_INDEX, a table entry outside [0, num_blocks)
 *                sets ATTN_DEVERR_BLOCK_TABLE; that token is not written.
 * Two tokens naming the same slot: which one lands is unspecified.
 */
ATTN_API attn_status paged_kv_append(const void *k_new, const void *v_new, const int32_t *seq_ids,
                                     const int32_t *positions, int num_tokens, const int32_t *block_table,
                                     int num_seqs, int max_blocks_per_seq, void *k_cache, void *v_cache,
                                     int num_blocks, int H, int d, int block_size, attn_dtype dt,
                                     int32_t *err_flag, attn_stream_t stream);

/*
 * Copy physical blocks for copy-on-write ("一文掌握大模型推理加速：
 * FlashAttention与PagedAttention技术详解", section 三 内存共享机制: before a
 * sequence writes into a block it shares, the block is copied to a new one
 * and that sequence's table entry is redirected -- the table update and the
 * reference counts are the caller's).
 *
 * For each pair i: block dst_blocks[i] of k_cache and of v_cache becomes a
 * copy of block src_blocks[i] (all heads, all slots).  The destination
 * blocks must be distinct and must not be sources of other pairs (the pairs
 * run concurrently).  Caches [num_blocks, H, block_size, d] of `dt`.
 * Supported    : ATTN_BF16 or ATTN_F32; d in {64, 128}; block_size in {16, 32}.
 * Device checks: an id outside [0, num_blocks) sets ATTN_DEVERR_BLOCK_TABLE
 *                and that pair is skipped.
 */
ATTN_API attn_status paged_block_copy(void *k_cache, void *v_cache, const int32_t *src_blocks,
                                      const int32_t *dst_blocks, int num_pairs, int num_blocks, int H, int d,
                                      int block_size, attn_dtype dt, int32_t *err_flag, attn_stream_t stream);

/*
 * Copy-on-write planning on the host: the table and reference-count half of
 * copying a shared block before a sequence writes into it
 * ("一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解", section 三
 * 内存共享机制: shared blocks carry a reference count; a write to a block
 * whose count is above 1 first copies it to a free block, the writer's table
 * entry is redirected to the copy and the counts are adjusted; the other
 * sharers keep the old contents).  The copies it plans are then made on the
 * device by paged_block_copy, before the writes (paged_kv_append).
 *
 * All arrays are HOST memory owned by the caller; nothing is allocated and
 * no device call is made.
 * block_table  : int32 [num_seqs, max_blocks_per_seq], edited in place:
 *                the entries of copied blocks point at their copies.
 * ref_counts   : int32 [num_blocks], edited in place (sharers per block).
 * free_list    : int32 [*free_count], a stack of free block ids (count 0):
 *                copies take blocks from its end; *free_count is updated.
 * write_seqs,
 * write_blocks : int32 [num_writes]: the pending writes, (sequence, logical
 *                block), in the order they happen.  A write whose block has
 *                count 1 is the writer's own (no copy); a repeated write, or
 *                the last sharer's write, finds its block exclusive.
 * src_out,
 * dst_out      : int32 [num_writes] (capacity): the copy pairs, in order;
 * *num_copies  : how many were written (0 .. num_writes).
 * Errors: ATTN_EINVAL for a NULL pointer or negative size, a write outside
 *         the table, an entry with no block (< 0) or outside
 *         [0, num_blocks), a referenced block with a count below 1, or a
 *         "free" block out of range or still referenced; ATTN_ENOBLOCKS when
 *         the free list runs out.  On any error every array is left as it
 *         was (the batch is all or nothing) and *num_copies is 0.
 */
ATTN_API attn_status paged_cow_plan(int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                                    int32_t *ref_counts, int num_blocks, int32_t *free_list, int32_t *free_count,
                                    const int32_t *write_seqs, const int32_t *write_blocks, int num_writes,
                                    int32_t *src_out, int32_t *dst_out, int32_t *num_copies);

/*
 * Synchronise `stream`, read the device int32 at err_flag and return
 * ATTN_OK if it is 0, ATTN_EDEVICE otherwise (the bits are written to
 * *bits_out when it is not NULL).  The flag is not reset.
 */
ATTN_API attn_status attn_read_error(const int32_t *err_flag, int32_t *bits_out, attn_stream_t stream);

/*
 * Self-test of the failure path shared by every pipeline wait: launches one
 * 32-thread CTA that waits, through the same bounded wait the kernels use,
 * on an mbarrier phase that nothing completes.  After the wait limit (1 s of
 * wall clock) the wait ORs ATTN_DEVERR_TIMEOUT into *err_flag (device int32,
 * required) and gives up; *result (device int32, may be NULL) is set to 0 for
 * "gave up", 1 for "completed" (never, here).  The kernel then returns
 * normally, so the context stays usable.  Asynchronous on `stream`; for
 * tests of error reporting (read the flag with attn_read_error).
 * Errors: ATTN_EINVAL for a NULL or misaligned err_flag or result.
 */
ATTN_API attn_status attn_selftest_wait_timeout(int32_t *err_flag, int32_t *result, attn_stream_t stream);

/*
 * Self-test of the exponential the bf16 prefill kernel computes on the FMA
 * pipe for part of each score row (FlashAttention-3's "softmax under the
 * asynchronous GEMMs" needs the exponentials to keep pace with the tensor
 * cores: "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解",
 * section 二 FlashAttention-3改进).  y[i] = the kernel's 2^x[i] for
 * i < n: a cubic in f = x - round(x) with round(x) added to the exponent,
 * x clamped to >= -125.  The stated bound is a relative error <= 7.5e-5
 * over [-125, 8], the kernel's range.
 *
 * x, y : device fp32 arrays of n elements (4-byte aligned; they may not
 *        overlap).  Asynchronous on `stream`.
 * Errors: ATTN_EINVAL for n < 0 or a NULL / misaligned pointer (n > 0).
 */
ATTN_API attn_status attn_selftest_exp2_poly(const float *x, float *y, int n, attn_stream_t stream);

/* Static, human-readable name of a status code. */
ATTN_API const char *attn_status_str(attn_status s);

#ifdef __cplusplus
}
#endif

#endif /* ONLINE_SOFTMAX_PAGED_ATTN_H */
