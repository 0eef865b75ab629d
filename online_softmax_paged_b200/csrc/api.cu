// api.cu -- the extern "C" boundary declared in include/attn.h: argument
// checks, dispatch to the sm_100a kernels, status codes.  No allocation, no
// host synchronisation (except attn_read_error, which exists to sync).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/attn.h"
#include "launch.h"

namespace osp {
// One CTA waits on an mbarrier phase that never completes (selftest.cu).
attn_status launch_wait_timeout_selftest(int32_t *err_flag, int32_t *result, cudaStream_t stream);
// The prefill softmax's FMA-pipe 2^x on given inputs (selftest.cu).
attn_status launch_exp2_poly_selftest(const float *x, float *y, int n, cudaStream_t stream);
}  // namespace osp

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

attn_status attn_fwd(const void *Q, const void *K, const void *V, void *O, float *LSE, int B, int H, int N, int d,
                     int causal, float scale, attn_dtype dt, int32_t *err_flag, attn_stream_t stream) {
    if (!Q || !K || !V || !O || !LSE) return ATTN_EINVAL;
    if (B < 1 || H < 1 || N < 1) return ATTN_EINVAL;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_EINVAL;
    if (dt != ATTN_F32 && dt != ATTN_BF16) return ATTN_EINVAL;
    if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return ATTN_EINVAL;
    if ((long long)B * H > 0x7fffffffLL / 2) return ATTN_EINVAL;
    if (dt == ATTN_F32 && (H > 65535 || B > 65535)) return ATTN_EINVAL;
    osp::DenseLaunch p{Q, K, V, O, LSE, B, H, N, d, causal ? 1 : 0, scale, err_flag};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dt == ATTN_BF16 ? osp::launch_prefill_bf16(p, s) : osp::launch_dense_f32(p, s);
}

attn_status attn_quantize_fp8(const void *x, void *codes, float *scales, int BH, int N, int d, const int8_t *signs,
                              attn_stream_t stream) {
    if (BH < 0 || N < 0) return ATTN_EINVAL;
    if (d != 128) return ATTN_EUNSUPPORTED;
    if (BH == 0 || N == 0) return ATTN_OK;
    if (!x || !codes || !scales) return ATTN_EINVAL;
    if (!aligned16(x) || !aligned16(codes) || ((uintptr_t)scales & 3u)) return ATTN_EINVAL;
    osp::QuantLaunch p{x, codes, scales, signs, BH, N};
    return osp::launch_quantize_fp8(p, reinterpret_cast<cudaStream_t>(stream));
}

attn_status attn_fwd_fp8(const void *q8, const float *q_scale, const void *k8, const float *k_scale, const void *V,
                         void *O, float *LSE, int B, int H, int N, int d, int causal, float scale, int32_t *err_flag,
                         attn_stream_t stream) {
    if (!q8 || !q_scale || !k8 || !k_scale || !V || !O || !LSE) return ATTN_EINVAL;
    if (B < 1 || H < 1 || N < 1) return ATTN_EINVAL;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_EINVAL;
    if (d != 128) return ATTN_EUNSUPPORTED;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(V) || !aligned16(O) || ((uintptr_t)LSE & 3u) ||
        ((uintptr_t)q_scale & 3u) || ((uintptr_t)k_scale & 3u))
        return ATTN_EINVAL;
    if ((long long)B * H > 0x7fffffffLL / 2) return ATTN_EINVAL;
    osp::Fp8Launch p{q8, k8, V, q_scale, k_scale, O, LSE, B, H, N, causal ? 1 : 0, scale, err_flag};
    return osp::launch_prefill_fp8(p, reinterpret_cast<cudaStream_t>(stream));
}

size_t paged_attn_decode_workspace_size(int num_seqs, int H, int d, int max_blocks_per_seq, int block_size) {
    if (num_seqs < 0 || H < 1 || d != 128 || max_blocks_per_seq < 1 || block_size < 16 || block_size % 16)
        return 0;
    return osp::decode_workspace_bytes(num_seqs, H, H, d, max_blocks_per_seq, block_size);
}

size_t paged_attn_decode_gqa_workspace_size(int num_seqs, int H_q, int H_kv, int d, int max_blocks_per_seq,
                                            int block_size) {
    if (num_seqs < 0 || H_q < 1 || H_kv < 1 || H_q % H_kv || d != 128 || max_blocks_per_seq < 1 ||
        block_size < 16 || block_size % 16)
        return 0;
    return osp::decode_workspace_bytes(num_seqs, H_q, H_kv, d, max_blocks_per_seq, block_size);
}

int paged_attn_decode_split_tokens(int num_seqs, int H, int d, int max_blocks_per_seq, int block_size) {
    if (num_seqs < 0 || H < 1 || d != 128 || max_blocks_per_seq < 1 || block_size < 16 || block_size % 16)
        return 0;
    return osp::decode_split_tokens(num_seqs, H, H, d, max_blocks_per_seq, block_size);
}

namespace {

attn_status decode_impl(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                        const int32_t *seq_lens, int block_size, void *O, float *LSE, int num_seqs, int H, int Hkv,
                        int d, int num_blocks, int max_blocks_per_seq, float scale, attn_dtype dt, void *workspace,
                        size_t workspace_bytes, int32_t *err_flag, attn_stream_t stream) {
    if (dt != ATTN_F32 && dt != ATTN_BF16) return ATTN_EINVAL;
    if (num_seqs < 0 || H < 1 || Hkv < 1 || num_blocks < 1 || max_blocks_per_seq < 1) return ATTN_EINVAL;
    if (H % Hkv) return ATTN_EINVAL;
    const int G = H / Hkv;
    if (G != 1 && G != 2 && G != 4 && G % 8 != 0) return ATTN_EUNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_EINVAL;
    if (dt != ATTN_BF16) return ATTN_EUNSUPPORTED;
    if (d != 128) return ATTN_EUNSUPPORTED;
    if (block_size != 16 && block_size != 32) return ATTN_EUNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size > 0x7fffffffLL) return ATTN_EINVAL;
    if ((long long)num_blocks * Hkv * block_size * d > (1LL << 46)) return ATTN_EINVAL;
    if (num_seqs == 0) return ATTN_OK;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !O || !LSE || !workspace) return ATTN_EINVAL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(O) || !aligned16(workspace))
        return ATTN_EINVAL;
    if (((uintptr_t)block_table & 3u) || ((uintptr_t)seq_lens & 3u) || ((uintptr_t)LSE & 3u)) return ATTN_EINVAL;
    if ((long long)num_seqs * H > 0x7fffffffLL / 4) return ATTN_EINVAL;
    if (workspace_bytes < osp::decode_workspace_bytes(num_seqs, H, Hkv, d, max_blocks_per_seq, block_size))
        return ATTN_EINVAL;
    osp::DecodeLaunch p{q,        k_cache,  v_cache, block_table, seq_lens,         O,          LSE,
                        num_seqs, H,        d,       num_blocks,  max_blocks_per_seq, block_size, scale,
                        workspace, err_flag, Hkv};
    return osp::launch_paged_decode(p, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

attn_status paged_attn_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                              const int32_t *seq_lens, int block_size, void *O, float *LSE, int num_seqs, int H,
                              int d, int num_blocks, int max_blocks_per_seq, float scale, attn_dtype dt,
                              void *workspace, size_t workspace_bytes, int32_t *err_flag, attn_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE, num_seqs, H, H, d,
                       num_blocks, max_blocks_per_seq, scale, dt, workspace, workspace_bytes, err_flag, stream);
}

attn_status paged_attn_decode_gqa(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, const int32_t *seq_lens, int block_size, void *O,
                                  float *LSE, int num_seqs, int H_q, int H_kv, int d, int num_blocks,
                                  int max_blocks_per_seq, float scale, attn_dtype dt, void *workspace,
                                  size_t workspace_bytes, int32_t *err_flag, attn_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE, num_seqs, H_q, H_kv, d,
                       num_blocks, max_blocks_per_seq, scale, dt, workspace, workspace_bytes, err_flag, stream);
}

attn_status paged_attn_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                               const int32_t *seq_lens, const int32_t *cu_q, int block_size, void *O, float *LSE,
                               int num_seqs, int total_q, int max_q_per_seq, int H_q, int H_kv, int d, int num_blocks,
                               int max_blocks_per_seq, float scale, attn_dtype dt, int32_t *err_flag,
                               attn_stream_t stream) {
    if (dt != ATTN_F32 && dt != ATTN_BF16) return ATTN_EINVAL;
    if (num_seqs < 0 || total_q < 0 || max_q_per_seq < 0 || H_q < 1 || H_kv < 1 || num_blocks < 1 ||
        max_blocks_per_seq < 1)
        return ATTN_EINVAL;
    if (H_q % H_kv) return ATTN_EINVAL;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_EINVAL;
    if (dt != ATTN_BF16) return ATTN_EUNSUPPORTED;
    if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
    if (block_size != 16 && block_size != 32) return ATTN_EUNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size > 0x7fffffffLL) return ATTN_EINVAL;
    if ((long long)num_blocks * H_kv * block_size > 0x7fffffffLL) return ATTN_EINVAL;
    if ((long long)total_q * H_q > 0x7fffffffLL || (long long)num_seqs * H_q > 0x7fffffffLL / 64) return ATTN_EINVAL;
    if (num_seqs == 0 || total_q == 0 || max_q_per_seq == 0) return ATTN_OK;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !cu_q || !O || !LSE) return ATTN_EINVAL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(O)) return ATTN_EINVAL;
    if (((uintptr_t)block_table & 3u) || ((uintptr_t)seq_lens & 3u) || ((uintptr_t)cu_q & 3u) ||
        ((uintptr_t)LSE & 3u))
        return ATTN_EINVAL;
    osp::PagedPrefillLaunch p{q,       k_cache, v_cache, block_table, seq_lens,   cu_q,               O,
                              LSE,     num_seqs, total_q, max_q_per_seq, H_q,      H_kv,              d,
                              num_blocks, max_blocks_per_seq, block_size, scale,   err_flag};
    return osp::launch_paged_prefill(p, reinterpret_cast<cudaStream_t>(stream));
}

attn_status paged_kv_append(const void *k_new, const void *v_new, const int32_t *seq_ids, const int32_t *positions,
                            int num_tokens, const int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                            void *k_cache, void *v_cache, int num_blocks, int H, int d, int block_size,
                            attn_dtype dt, int32_t *err_flag, attn_stream_t stream) {
    if (dt != ATTN_F32 && dt != ATTN_BF16) return ATTN_EINVAL;
    if (num_tokens < 0 || num_seqs < 1 || max_blocks_per_seq < 1 || num_blocks < 1 || H < 1) return ATTN_EINVAL;
    if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
    if (block_size != 16 && block_size != 32) return ATTN_EUNSUPPORTED;
    if ((long long)max_blocks_per_seq * block_size > 0x7fffffffLL) return ATTN_EINVAL;
    if (num_tokens == 0) return ATTN_OK;
    if (!k_new || !v_new || !seq_ids || !positions || !block_table || !k_cache || !v_cache) return ATTN_EINVAL;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) return ATTN_EINVAL;
    if (((uintptr_t)seq_ids & 3u) || ((uintptr_t)positions & 3u) || ((uintptr_t)block_table & 3u)) return ATTN_EINVAL;
    osp::AppendLaunch p{k_new,      v_new, seq_ids, positions, block_table, k_cache, v_cache, num_tokens, num_seqs,
                        max_blocks_per_seq, num_blocks, H, d, block_size, dt == ATTN_BF16 ? 2 : 4, err_flag};
    return osp::launch_kv_append(p, reinterpret_cast<cudaStream_t>(stream));
}

attn_status paged_block_copy(void *k_cache, void *v_cache, const int32_t *src_blocks, const int32_t *dst_blocks,
                             int num_pairs, int num_blocks, int H, int d, int block_size, attn_dtype dt,
                             int32_t *err_flag, attn_stream_t stream) {
    if (dt != ATTN_F32 && dt != ATTN_BF16) return ATTN_EINVAL;
    if (num_pairs < 0 || num_blocks < 1 || H < 1) return ATTN_EINVAL;
    if (d != 64 && d != 128) return ATTN_EUNSUPPORTED;
    if (block_size != 16 && block_size != 32) return ATTN_EUNSUPPORTED;
    if (num_pairs > 0x7fffffff / 2) return ATTN_EINVAL;
    if (num_pairs == 0) return ATTN_OK;
    if (!k_cache || !v_cache || !src_blocks || !dst_blocks) return ATTN_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return ATTN_EINVAL;
    if (((uintptr_t)src_blocks & 3u) || ((uintptr_t)dst_blocks & 3u)) return ATTN_EINVAL;
    osp::CopyLaunch p{k_cache, v_cache, src_blocks, dst_blocks, num_pairs, num_blocks, H, d, block_size,
                      dt == ATTN_BF16 ? 2 : 4, err_flag};
    return osp::launch_block_copy(p, reinterpret_cast<cudaStream_t>(stream));
}

attn_status attn_selftest_wait_timeout(int32_t *err_flag, int32_t *result, attn_stream_t stream) {
    if (!err_flag || ((uintptr_t)err_flag & 3u) || ((uintptr_t)result & 3u)) return ATTN_EINVAL;
    return osp::launch_wait_timeout_selftest(err_flag, result, reinterpret_cast<cudaStream_t>(stream));
}

attn_status attn_selftest_exp2_poly(const float *x, float *y, int n, attn_stream_t stream) {
    if (n < 0) return ATTN_EINVAL;
    if (n == 0) return ATTN_OK;
    if (!x || !y || ((uintptr_t)x & 3u) || ((uintptr_t)y & 3u)) return ATTN_EINVAL;
    return osp::launch_exp2_poly_selftest(x, y, n, reinterpret_cast<cudaStream_t>(stream));
}

attn_status attn_read_error(const int32_t *err_flag, int32_t *bits_out, attn_stream_t stream) {
    if (!err_flag) return ATTN_EINVAL;
    int32_t v = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, err_flag, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ATTN_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ECUDA;
    if (bits_out) *bits_out = v;
    return v ? ATTN_EDEVICE : ATTN_OK;
}

const char *attn_status_str(attn_status s) {
    switch (s) {
        case ATTN_OK: return "ok";
        case ATTN_EINVAL: return "invalid argument";
        case ATTN_EUNSUPPORTED: return "unsupported configuration";
        case ATTN_ECUDA: return "CUDA error";
        case ATTN_EDEVICE: return "device-side error reported in err_flag";
        case ATTN_ENOBLOCKS: return "no free block left for a copy-on-write copy";
    }
    return "unknown status";
}

}  // extern "C"
