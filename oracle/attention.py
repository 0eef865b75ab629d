"""fp64 CPU oracle for exact attention forward, dense and paged.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
legs of ``bench.py`` may call it.  It shares no code with the CUDA path.

Sources (the web pages this build follows; titles as printed):

* [技术详解] "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
  (devpress.csdn.net) -- §一 (standard self-attention formula and its O(n²)
  cost), §二 "核心原理" (tiling, safe softmax, stored statistics m and
  logsumexp), §二 "FlashAttention-2 改进" (store only logsumexp), §三
  "核心原理" (block table: contiguous logical blocks, non-contiguous
  physical blocks of 16 or 32 tokens).
* [区别] "FlashAttention 和 PagedAttention 有什么区别？" (mstx.cn) -- Q1
  (online softmax keeps a running max and normaliser; exact, not approximate),
  Q2 comparison table (paging changes storage only, not the attention math).
* [实现解析] "第 2 章核心模块：FlashAttention-2 与 PagedAttention 实现解析"
  (aiknowledge.cn) -- §2.1 design two (incremental normalisation: update the
  running max m and sum l per K tile and correct the accumulated O; provably
  equal to one-shot softmax), §2.2 (the paged loop: per logical block look up
  the physical block, fetch its K/V, score, merge into the running max/sum).
* [内存优化] "Transformer内存优化：从Flash Attention到Page Attention"
  (trdm.cn) -- §1.1 (tensor layout [batch, heads, seq_len, dim]), §2.1 (the
  q-block / k-block tile loop).

Readings where the pages are silent or garbled (the formula itself was an
image and is lost from [技术详解] §一):

1. Attention is O = softmax(S) V with S = scale * Q K^T, scale = 1/sqrt(d)
   unless the caller passes another value.
2. LSE is the natural log of sum_j exp(s_ij), scale included.
3. Causal means key j is visible to query i iff j <= i (square, Nq = Nk).
4. Paged decode: seq_lens[s] counts every key the single query attends to;
   no mask inside [0, L).  L = 0 gives O = 0 and LSE = -inf.
5. Split-KV merge (not on the pages): LSE = log sum_p exp(LSE_p) and
   O = sum_p exp(LSE_p - LSE) O_p, which follows from the statistics the pages
   keep (m, l and logsumexp).

Every array is float64; callers upcast bf16/fp32 inputs exactly.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -math.inf


def _visible(i0: int, i1: int, n_keys: int, causal: bool) -> np.ndarray:
    """Boolean mask [i1-i0, n_keys]: key j visible to query row i.

    Reading 3 above; [技术详解] §一 for the full (non-causal) row.
    """
    rows = np.arange(i0, i1)[:, None]
    cols = np.arange(n_keys)[None, :]
    if causal:
        return cols <= rows
    return np.ones((i1 - i0, n_keys), dtype=bool)


def scores(Q: np.ndarray, K: np.ndarray, scale: float) -> np.ndarray:
    """s_ij = scale * <q_i, k_j> for one head: Q [Nq, d], K [Nk, d] -> [Nq, Nk].

    [技术详解] §一 (QK^T / sqrt(d_k)); reading 1.
    """
    return scale * (Q @ K.T)


def softmax_probs(Q, K, causal: bool, scale: float) -> np.ndarray:
    """Materialised probability matrix P for one head (the N x N matrix the
    standard method stores, [技术详解] §一 / [区别] Q1).

    Safe softmax: subtract the row max before exponentiating ([技术详解] §二
    "核心原理").  Masked entries are exactly 0.
    """
    S = scores(Q, K, scale)
    vis = _visible(0, Q.shape[0], K.shape[0], causal)
    S = np.where(vis, S, NEG_INF)
    m = S.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    P = np.exp(S - m)
    P = np.where(vis, P, 0.0)
    l = P.sum(axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(l > 0, P / l, 0.0)


def attention_head(Q, K, V, causal: bool, scale: float, row_chunk: int = 1024):
    """Exact attention for one head by the plain definition.

    Q [Nq, d], K [Nk, d], V [Nk, dv] -> O [Nq, dv], LSE [Nq].
    Full score rows are materialised, ``row_chunk`` query rows at a time (the
    chunking only bounds host memory; every row is computed in one shot).

    LSE_i = m_i + ln sum_j exp(s_ij - m_i)   (reading 2; [技术详解] §二 stores
    m and logsumexp, "FlashAttention-2 改进" stores only logsumexp)
    O_i   = sum_j exp(s_ij - LSE_i) v_j
    A row with no visible key gives O = 0, LSE = -inf (reading 4).
    """
    Nq = Q.shape[0]
    O = np.zeros((Nq, V.shape[1]), dtype=np.float64)
    LSE = np.full((Nq,), NEG_INF, dtype=np.float64)
    for i0 in range(0, Nq, row_chunk):
        i1 = min(Nq, i0 + row_chunk)
        S = scores(Q[i0:i1], K, scale)
        vis = _visible(i0, i1, K.shape[0], causal)
        S = np.where(vis, S, NEG_INF)
        m = S.max(axis=1) if S.shape[1] else np.full((i1 - i0,), NEG_INF)
        finite = np.isfinite(m)
        m_safe = np.where(finite, m, 0.0)
        P = np.where(vis, np.exp(S - m_safe[:, None]), 0.0)
        l = P.sum(axis=1)
        ok = l > 0
        with np.errstate(divide="ignore", invalid="ignore"):
            LSE[i0:i1] = np.where(ok, m_safe + np.log(np.where(ok, l, 1.0)), NEG_INF)
            O[i0:i1] = np.where(ok[:, None], (P @ V) / np.where(ok, l, 1.0)[:, None], 0.0)
    return O, LSE


def attention_dense(Q, K, V, causal: bool, scale: float, heads=None, row_chunk: int = 1024):
    """Dense prefill oracle over [B, H, N, d] arrays ([内存优化] §1.1 layout).

    Returns O [B, H, N, d] and LSE [B, H, N] (float64).  ``heads`` optionally
    restricts the work to a list of (b, h) pairs; the other entries stay
    NaN so that a caller cannot mistake them for results.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, N, _ = Q.shape
    O = np.full(Q.shape[:3] + (V.shape[3],), np.nan)
    LSE = np.full((B, H, N), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in todo:
        O[b, h], LSE[b, h] = attention_head(Q[b, h], K[b, h], V[b, h], causal, scale, row_chunk)
    return O, LSE


def attention_online_tiled(Q, K, V, causal: bool, scale: float, Br: int, Bc: int):
    """The method's own tile loop for one head, in the pages' order.

    [实现解析] §2.1 designs one and two, [技术详解] §二 "分块策略", [内存优化]
    §2.1: Q is cut into row tiles of Br rows and K/V into column tiles of Bc
    rows.  For each Q tile a running max m and running sum l are kept per row;
    each new K/V tile j gives scores S_j, then

        m_new = max(m, rowmax(S_j))
        l     = exp(m - m_new) * l + rowsum(exp(S_j - m_new))
        O     = exp(m - m_new) * O + exp(S_j - m_new) V_j
        m     = m_new

    and after the last tile O /= l and LSE = m + ln l.  No blocking beyond
    this; the result must equal :func:`attention_head` (the pages call the two
    mathematically equivalent).
    """
    Nq, Nk = Q.shape[0], K.shape[0]
    O_out = np.zeros((Nq, V.shape[1]))
    LSE_out = np.full((Nq,), NEG_INF)
    for i0 in range(0, Nq, Br):
        i1 = min(Nq, i0 + Br)
        m = np.full((i1 - i0,), NEG_INF)
        l = np.zeros((i1 - i0,))
        acc = np.zeros((i1 - i0, V.shape[1]))
        for j0 in range(0, Nk, Bc):
            j1 = min(Nk, j0 + Bc)
            S = scale * (Q[i0:i1] @ K[j0:j1].T)
            if causal:
                rows = np.arange(i0, i1)[:, None]
                cols = np.arange(j0, j1)[None, :]
                S = np.where(cols <= rows, S, NEG_INF)
            m_new = np.maximum(m, S.max(axis=1))
            # rows that have seen no visible key yet keep m = -inf
            live = np.isfinite(m_new)
            m_safe = np.where(live, m_new, 0.0)
            alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
            P = np.where(np.isfinite(S), np.exp(S - m_safe[:, None]), 0.0)
            l = alpha * l + P.sum(axis=1)
            acc = alpha[:, None] * acc + P @ V[j0:j1]
            m = m_new
        ok = l > 0
        with np.errstate(divide="ignore", invalid="ignore"):
            O_out[i0:i1] = np.where(ok[:, None], acc / np.where(ok, l, 1.0)[:, None], 0.0)
            LSE_out[i0:i1] = np.where(ok, m + np.log(np.where(ok, l, 1.0)), NEG_INF)
    return O_out, LSE_out


def gather_paged(cache, block_table_row, L: int, block_size: int) -> np.ndarray:
    """Resolve one sequence's block table by explicit copy.

    [技术详解] §三 "核心原理" (block table maps contiguous logical blocks to
    non-contiguous physical blocks), [实现解析] §2.2 (phys = block_table[lb];
    fetch that block).  cache is [num_blocks, H, block_size, d]; the result is
    the contiguous [H, L, d] sequence.  An entry outside [0, num_blocks)
    among the first ceil(L / block_size) raises IndexError.
    """
    n_blk = -(-L // block_size)
    num_blocks = cache.shape[0]
    parts = []
    for lb in range(n_blk):
        phys = int(block_table_row[lb])
        if phys < 0 or phys >= num_blocks:
            raise IndexError(f"block_table entry {phys} for logical block {lb} outside [0, {num_blocks})")
        parts.append(np.asarray(cache[phys], dtype=np.float64))
    if not parts:
        return np.zeros((cache.shape[1], 0, cache.shape[3]))
    return np.concatenate(parts, axis=1)[:, :L, :]


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, block_size: int, scale: float, seqs=None):
    """Paged decode oracle: one query token per sequence.

    q [S, Hq, d]; caches [num_blocks, Hkv, block_size, d] with Hq a multiple
    of Hkv (query head h reads key/value head h // (Hq / Hkv): grouped-query
    attention; Hq == Hkv is plain multi-head attention); block_table
    [S, max_blocks_per_seq]; seq_lens [S].  For each sequence the keys and
    values are first copied into contiguous [Hkv, L, d] arrays
    (:func:`gather_paged`), then the dense definition runs with one query row
    and no mask ([区别] Q2: paging changes storage, not the math; reading 4).
    Returns O [S, Hq, d], LSE [S, Hq]; sequences not in ``seqs`` stay NaN.
    """
    S, H, d = q.shape
    Hkv = k_cache.shape[1]
    if H % Hkv:
        raise ValueError("query heads must be a multiple of key/value heads")
    G = H // Hkv
    O = np.full((S, H, v_cache.shape[3]), np.nan)
    LSE = np.full((S, H), np.nan)
    for s in (range(S) if seqs is None else seqs):
        L = int(seq_lens[s])
        Ks = gather_paged(k_cache, block_table[s], L, block_size)
        Vs = gather_paged(v_cache, block_table[s], L, block_size)
        for h in range(H):
            o, lse = attention_head(np.asarray(q[s, h:h + 1], dtype=np.float64), Ks[h // G], Vs[h // G], False,
                                    scale)
            O[s, h] = o[0]
            LSE[s, h] = lse[0]
    return O, LSE


def merge_partials(O_parts: np.ndarray, LSE_parts: np.ndarray):
    """Combine attention over disjoint key subsets (split-KV merge).

    O_parts [P, ..., d], LSE_parts [P, ...] -> O [..., d], LSE [...]:
        LSE = ln sum_p exp(LSE_p),  O = sum_p exp(LSE_p - LSE) O_p.
    Reading 5: this follows from keeping (m, l) / logsumexp per row
    ([技术详解] §二 "核心原理", [实现解析] §2.1).  Parts with LSE_p = -inf
    contribute nothing; all parts -inf gives O = 0, LSE = -inf.
    """
    O_parts = np.asarray(O_parts, dtype=np.float64)
    LSE_parts = np.asarray(LSE_parts, dtype=np.float64)
    m = LSE_parts.max(axis=0)
    live = np.isfinite(m)
    m_safe = np.where(live, m, 0.0)
    w = np.where(np.isfinite(LSE_parts), np.exp(LSE_parts - m_safe), 0.0)
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        LSE = np.where(live, m_safe + np.log(np.where(live, tot, 1.0)), NEG_INF)
        O = np.where(live[..., None], (w[..., None] * O_parts).sum(axis=0) / np.where(live, tot, 1.0)[..., None], 0.0)
    return O, LSE


def attention_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Algorithmic FLOPs of one prefill call: two contractions of 2*d flops per
    visible (query, key) pair; causal counts the lower triangle with the
    diagonal, N(N+1)/2 pairs per head ([技术详解] §一: O(n^2 d) time)."""
    pairs = N * (N + 1) // 2 if causal else N * N
    return 4.0 * B * H * d * pairs


def kv_append(k_cache, v_cache, block_table, k_new, v_new, seq_ids, positions, block_size: int):
    """Write new tokens' keys/values into the paged cache (copy; float64 or any
    dtype is kept).

    [技术详解] §三 "核心原理" (a new token goes into the sequence's current
    block, found through its block table) and [实现解析] §2.2 (logical block
    -> physical block).  Token t of sequence seq_ids[t] at position
    positions[t] lands in physical block block_table[s][pos // block_size],
    slot pos % block_size, for every head.  Returns new arrays; a token whose
    sequence, position or table entry is out of range is skipped and reported
    in the returned list of skipped token indices.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    num_blocks = k_out.shape[0]
    S, mb = np.asarray(block_table).shape
    skipped = []
    for t in range(len(seq_ids)):
        s, pos = int(seq_ids[t]), int(positions[t])
        if not (0 <= s < S and 0 <= pos < mb * block_size):
            skipped.append(t)
            continue
        phys = int(block_table[s][pos // block_size])
        if not (0 <= phys < num_blocks):
            skipped.append(t)
            continue
        k_out[phys, :, pos % block_size, :] = k_new[t]
        v_out[phys, :, pos % block_size, :] = v_new[t]
    return k_out, v_out, skipped


def block_copy(k_cache, v_cache, src_blocks, dst_blocks):
    """Copy-on-write step: physical block src -> dst (all heads, all slots) for
    each pair, in pair order ([技术详解] §三 内存共享机制: a write to a shared
    block first copies it to a new block).  Pairs with an id out of range are
    skipped and reported."""
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    n = k_out.shape[0]
    skipped = []
    for i, (a, b) in enumerate(zip(src_blocks, dst_blocks)):
        a, b = int(a), int(b)
        if not (0 <= a < n and 0 <= b < n):
            skipped.append(i)
            continue
        k_out[b] = k_cache[a]
        v_out[b] = v_cache[a]
    return k_out, v_out, skipped


def cow_plan(block_table, ref_counts, free_list, writes):
    """Copy-on-write planning for a batch of pending writes.

    [技术详解] §三 "内存共享机制": blocks shared by several sequences carry a
    reference count; before a sequence writes into a block whose count is
    above 1, the block is copied to a free block, the writer's table entry
    is pointed at the copy and the counts are adjusted, so the other
    sequences keep the old contents ([区别] Q2 and [实现解析] §2.2 give the
    table from logical to physical blocks this edits).

    block_table [S, max_blocks] (entries < 0: no block), ref_counts
    [num_blocks], free_list a stack of free block ids (taken from its end),
    writes a sequence of (seq, logical block) in the order they happen.
    Each write, in order: the block p = table[s][lb]; if ref[p] == 1 the
    sequence owns it and writes in place; otherwise the last free block f is
    taken, ref[p] -= 1, ref[f] = 1, table[s][lb] = f and the pair (p, f) is
    emitted (the copy runs before the write).  Returns new arrays (table,
    counts, free list) and the pairs as (src, dst) lists; the inputs are not
    modified.  Raises ValueError for a write outside the table, an entry
    without a block or outside [0, num_blocks), a referenced block with a
    count below 1, a free block that is out of range or still referenced,
    or a free list that runs out.
    """
    table = np.array(block_table, dtype=np.int64, copy=True)
    refs = np.array(ref_counts, dtype=np.int64, copy=True)
    free = [int(b) for b in free_list]
    S, mb = table.shape
    nb = refs.shape[0]
    src, dst = [], []
    for s, lb in writes:
        s, lb = int(s), int(lb)
        if not (0 <= s < S and 0 <= lb < mb):
            raise ValueError(f"write ({s}, {lb}) outside the table")
        p = int(table[s, lb])
        if not 0 <= p < nb:
            raise ValueError(f"write ({s}, {lb}): no block or block {p} out of range")
        if refs[p] < 1:
            raise ValueError(f"block {p} is referenced but its count is {refs[p]}")
        if refs[p] == 1:
            continue
        if not free:
            raise ValueError("the free list ran out")
        f = free.pop()
        if not 0 <= f < nb or refs[f] != 0:
            raise ValueError(f"free block {f} is out of range or still referenced")
        refs[p] -= 1
        refs[f] = 1
        table[s, lb] = f
        src.append(p)
        dst.append(f)
    return table, refs, free, src, dst


def paged_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_q, block_size: int, scale: float, seqs=None):
    """Multi-token paged prefill / append oracle.

    [实现解析] §2.2 runs its paged loop "for each query position i"; [实现解析]
    §2.3 and [区别] Q2 put PagedAttention's storage under FlashAttention's
    computation.  Sequence s has n_s = cu_q[s+1] - cu_q[s] new query tokens,
    the last n_s of its seq_lens[s] = L_s cached tokens (their keys/values
    are already in the cache).  Query token i sits at position
    L_s - n_s + i and attends keys 0 .. L_s - n_s + i (causal, offset by the
    cached prefix).  Keys/values are resolved by explicit copy
    (:func:`gather_paged`); query head h reads key/value head h // G
    (G = Hq / Hkv).  q [total_q, Hq, d] -> O [total_q, Hq, d], LSE [total_q, Hq];
    sequences not in ``seqs`` stay NaN.
    """
    T, H, d = q.shape
    Hkv = k_cache.shape[1]
    if H % Hkv:
        raise ValueError("query heads must be a multiple of key/value heads")
    G = H // Hkv
    O = np.full((T, H, v_cache.shape[3]), np.nan)
    LSE = np.full((T, H), np.nan)
    S = len(seq_lens)
    for s in (range(S) if seqs is None else seqs):
        q0, q1 = int(cu_q[s]), int(cu_q[s + 1])
        n, L = q1 - q0, int(seq_lens[s])
        if n == 0:
            continue
        if n > L:
            raise ValueError("a sequence has more new tokens than cached tokens")
        Ks = gather_paged(k_cache, block_table[s], L, block_size)
        Vs = gather_paged(v_cache, block_table[s], L, block_size)
        for h in range(H):
            for i in range(n):
                p = L - n + i
                o, lse = attention_head(np.asarray(q[q0 + i, h:h + 1], dtype=np.float64), Ks[h // G][:p + 1],
                                        Vs[h // G][:p + 1], False, scale)
                O[q0 + i, h] = o[0]
                LSE[q0 + i, h] = lse[0]
    return O, LSE
