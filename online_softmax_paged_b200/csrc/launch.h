// launch.h -- internal launcher interface between the C ABI (api.cu) and the
// kernel translation units.  Not installed; the public ABI is include/attn.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/attn.h"

namespace osp {

struct DenseLaunch {
    const void *Q, *K, *V;
    void *O;
    float *LSE;
    int B, H, N, d, causal;
    float scale;
    int32_t *err_flag;
};

struct DecodeLaunch {
    const void *q, *k_cache, *v_cache;
    const int32_t *block_table, *seq_lens;
    void *O;
    float *LSE;
    int num_seqs, H, d, num_blocks, max_blocks, block_size;
    float scale;
    void *workspace;
    int32_t *err_flag;
    int Hkv;  // key/value heads (H / Hkv in {1, 2, 4, 8})
};

struct AppendLaunch {
    const void *k_new, *v_new;
    const int32_t *seq_ids, *positions, *block_table;
    void *k_cache, *v_cache;
    int num_tokens, num_seqs, max_blocks, num_blocks, H, d, block_size, elem_bytes;
    int32_t *err_flag;
};

struct CopyLaunch {
    void *k_cache, *v_cache;
    const int32_t *src_blocks, *dst_blocks;
    int num_pairs, num_blocks, H, d, block_size, elem_bytes;
    int32_t *err_flag;
};

struct PagedPrefillLaunch {
    const void *q, *k_cache, *v_cache;
    const int32_t *block_table, *seq_lens, *cu_q;
    void *O;
    float *LSE;
    int num_seqs, total_q, max_q_per_seq, Hq, Hkv, d, num_blocks, max_blocks, block_size;
    float scale;
    int32_t *err_flag;
};

struct QuantLaunch {
    const void *x;        // bf16 [BH, N, d]
    void *codes;          // e4m3 [BH, N, d]
    float *scales;        // [BH, ceil(N / 128)]
    const int8_t *signs;  // d entries of +-1, or null (no rotation)
    int BH, N;
};

struct Fp8Launch {
    const void *q8, *k8, *V;
    const float *q_scale, *k_scale;
    void *O;
    float *LSE;
    int B, H, N, causal;
    float scale;
    int32_t *err_flag;
};

// 2-D bf16 tensor map over `rows` rows of `inner` elements (row pitch
// `pitch_elems`), box 64 x box_rows, 128-byte swizzle (prefill_sm100.cu).
bool make_tensor_map_2d_bf16(CUtensorMap *m, const void *base, long long inner, long long rows, long long pitch_elems,
                             int box_rows);

attn_status launch_dense_f32(const DenseLaunch &p, cudaStream_t stream);
attn_status launch_quantize_fp8(const QuantLaunch &p, cudaStream_t stream);
attn_status launch_prefill_fp8(const Fp8Launch &p, cudaStream_t stream);
attn_status launch_paged_prefill(const PagedPrefillLaunch &p, cudaStream_t stream);
attn_status launch_kv_append(const AppendLaunch &p, cudaStream_t stream);
attn_status launch_block_copy(const CopyLaunch &p, cudaStream_t stream);
attn_status launch_prefill_bf16(const DenseLaunch &p, cudaStream_t stream);
attn_status launch_paged_decode(const DecodeLaunch &p, cudaStream_t stream);

// H query heads over Hkv key/value heads (Hkv = H: multi-head)
int decode_split_tokens(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size);
int decode_max_splits(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size);
size_t decode_workspace_bytes(int num_seqs, int H, int Hkv, int d, int max_blocks, int block_size);

}  // namespace osp
