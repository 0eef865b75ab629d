/*
 * Triple-loop attention in double precision: a second, independently written
 * oracle used to cross-check the numpy oracle on tiny shapes.
 *
 * TEST INFRASTRUCTURE ONLY.  The CUDA library never links or calls this file;
 * only tests, smoke() and the bench's CPU-baseline leg may.
 *
 * Definition followed ("一文掌握大模型推理加速：FlashAttention与PagedAttention
 * 技术详解", section 一, standard self-attention; the formula image is lost,
 * read as O = softmax(scale * Q K^T) V):
 *   s_ij  = scale * sum_c q_ic k_jc           for visible j (j <= i if causal)
 *   m_i   = max_j s_ij                          (safe softmax, section 二)
 *   LSE_i = m_i + log sum_j exp(s_ij - m_i)
 *   O_ic  = sum_j exp(s_ij - LSE_i) v_jc
 * A row with no visible key gets O = 0 and LSE = -inf.
 *
 * Paged decode ("第 2 章核心模块：FlashAttention-2 与 PagedAttention 实现解析",
 * section 2.2): key j of sequence s lives in physical block
 * block_table[s][j / bs] at slot j % bs.
 */
#include <math.h>
#include <stdint.h>

static void one_row(const double *q, int n_vis, int d,
                    const double *(*key_at)(const void *, int),
                    const double *(*val_at)(const void *, int),
                    const void *ctx, double scale, double *o, double *lse)
{
    int c, j;
    double m = -INFINITY, l = 0.0;
    for (c = 0; c < d; ++c) o[c] = 0.0;
    if (n_vis <= 0) { *lse = -INFINITY; return; }
    for (j = 0; j < n_vis; ++j) {
        const double *k = key_at(ctx, j);
        double s = 0.0;
        for (c = 0; c < d; ++c) s += q[c] * k[c];
        s *= scale;
        if (s > m) m = s;
    }
    for (j = 0; j < n_vis; ++j) {
        const double *k = key_at(ctx, j);
        const double *v = val_at(ctx, j);
        double s = 0.0, p;
        for (c = 0; c < d; ++c) s += q[c] * k[c];
        p = exp(s * scale - m);
        l += p;
        for (c = 0; c < d; ++c) o[c] += p * v[c];
    }
    for (c = 0; c < d; ++c) o[c] /= l;
    *lse = m + log(l);
}

/* ---- dense: K, V are [N, d] for one head ---- */
typedef struct { const double *K, *V; int d; } dense_ctx;
static const double *dense_key(const void *p, int j) { const dense_ctx *c = p; return c->K + (long)j * c->d; }
static const double *dense_val(const void *p, int j) { const dense_ctx *c = p; return c->V + (long)j * c->d; }

/* Q, K, V, O: [B, H, N, d] row-major; LSE: [B, H, N]. */
void brute_attention(const double *Q, const double *K, const double *V,
                     double *O, double *LSE, int B, int H, int N, int d,
                     int causal, double scale)
{
    int bh, i;
    for (bh = 0; bh < B * H; ++bh) {
        dense_ctx ctx = { K + (long)bh * N * d, V + (long)bh * N * d, d };
        for (i = 0; i < N; ++i) {
            long r = (long)bh * N + i;
            one_row(Q + r * d, causal ? i + 1 : N, d, dense_key, dense_val, &ctx, scale,
                    O + r * d, LSE + r);
        }
    }
}

/* ---- paged: caches are [num_blocks, H, bs, d] ---- */
typedef struct {
    const double *kc, *vc; const int32_t *row; int H, h, bs, d;
} paged_ctx;
static const double *paged_at(const double *cache, const paged_ctx *c, int j)
{
    long phys = c->row[j / c->bs];
    return cache + (((phys * c->H + c->h) * c->bs) + (j % c->bs)) * (long)c->d;
}
static const double *paged_key(const void *p, int j) { const paged_ctx *c = p; return paged_at(c->kc, c, j); }
static const double *paged_val(const void *p, int j) { const paged_ctx *c = p; return paged_at(c->vc, c, j); }

/* q, O: [S, H, d]; LSE: [S, H]; block_table: [S, max_blocks]; entries are
 * trusted (the caller checks them). */
void brute_paged_decode(const double *q, const double *k_cache, const double *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        int block_size, double *O, double *LSE,
                        int S, int H, int d, int max_blocks, double scale)
{
    int s, h;
    for (s = 0; s < S; ++s) {
        for (h = 0; h < H; ++h) {
            paged_ctx ctx = { k_cache, v_cache, block_table + (long)s * max_blocks, H, h, block_size, d };
            long r = (long)s * H + h;
            one_row(q + r * d, seq_lens[s], d, paged_key, paged_val, &ctx, scale, O + r * d, LSE + r);
        }
    }
}
