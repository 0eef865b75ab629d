"""Seeded synthetic inputs for the dense-prefill and paged-decode workloads.

Shared by the tests, ``bench.py`` and ``__graft_entry__``; it holds none of
the attention arithmetic, only random draws and block-table construction.
Both the oracle and the CUDA library receive the tensors built here.

Recipe (one ``torch.Generator`` per workload, seeded, draws in the order
listed in each function; ``.to(torch.bfloat16)`` rounds to nearest even).
The stream depends on the generator's device: a CUDA generator and a CPU
generator with the same seed give different numbers, which does not matter
because every comparison hands the same tensors to both sides.

The page shapes follow "一文掌握大模型推理加速：FlashAttention与PagedAttention
技术详解" §三 "核心原理" (blocks of 16 or 32 tokens, contiguous logical
blocks, non-contiguous physical blocks) and "第 2 章核心模块：FlashAttention-2
与 PagedAttention 实现解析" §2.2 (block table per sequence).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# The five workloads of the hot path, named by what they are.
DENSE_F32_SMALL = dict(B=1, H=2, N=128, d=64, causal=False, dtype=torch.float32, mult=1.0)
PREFILL_CAUSAL_2K = dict(B=4, H=16, N=2048, d=128, causal=True, dtype=torch.bfloat16, mult=1.0)
PREFILL_CAUSAL_16K = dict(B=1, H=32, N=16384, d=128, causal=True, dtype=torch.bfloat16, mult=0.5)
DECODE_UNIFORM = dict(num_seqs=64, H=32, d=128, block_size=16, pool=20000, len_lo=128, len_hi=4096)
DECODE_SHARED_PREFIX = dict(num_seqs=256, H=32, d=128, block_size=32, pool=20000, median=1024,
                            sigma=1.0, len_lo=1, len_hi=8192, group=8, prefix_tokens=512)
# chunked prefill over a paged cache: each sequence appends a 2048-token
# chunk after a cached context of U{0..6144} tokens; 32 query heads over 8
# key/value heads
PREFILL_PAGED_CHUNKED = dict(num_seqs=8, Hq=32, Hkv=8, d=128, block_size=16, pool=20000, chunk=2048,
                             ctx_lo=0, ctx_hi=6144)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device, dtype, mult=1.0, chunk_rows=None):
    """N(0,1) fp32 draws (times ``mult``) rounded to ``dtype``.

    Large tensors are drawn ``chunk_rows`` leading rows at a time so that the
    fp32 temporary stays small; the chunking is part of the recipe.
    """
    out = torch.empty(shape, dtype=dtype, device=device)
    n0 = shape[0]
    step = n0 if chunk_rows is None else chunk_rows
    for r0 in range(0, n0, step):
        r1 = min(n0, r0 + step)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device, dtype=torch.float32)
        if mult != 1.0:
            x.mul_(mult)
        out[r0:r1] = x.to(dtype)
    return out


def dense_inputs(B, H, N, d, dtype=torch.bfloat16, mult=1.0, seed=0, device="cpu", causal=False):
    """Q, K, V [B, H, N, d], drawn in that order (each N(0,1) * mult)."""
    g = _gen(seed, device)
    chunk = max(1, (1 << 26) // max(1, H * N * d))
    Q = _normal((B, H, N, d), g, device, dtype, mult, chunk)
    K = _normal((B, H, N, d), g, device, dtype, mult, chunk)
    V = _normal((B, H, N, d), g, device, dtype, mult, chunk)
    return dict(Q=Q, K=K, V=V, B=B, H=H, N=N, d=d, causal=causal, scale=1.0 / math.sqrt(d))


@dataclass
class PagedInputs:
    q: torch.Tensor            # [S, H, d]
    k_cache: torch.Tensor      # [num_blocks, H, block_size, d]
    v_cache: torch.Tensor      # [num_blocks, H, block_size, d]
    block_table: torch.Tensor  # int32 [S, max_blocks_per_seq], unused entries -1
    seq_lens: torch.Tensor     # int32 [S]
    block_size: int
    scale: float
    shared_groups: list = field(default_factory=list)  # lists of sequence ids sharing a prefix

    @property
    def num_seqs(self):
        return self.q.shape[0]

    @property
    def H(self):
        return self.q.shape[1]

    @property
    def d(self):
        return self.q.shape[2]

    @property
    def num_blocks(self):
        return self.k_cache.shape[0]

    @property
    def max_blocks_per_seq(self):
        return self.block_table.shape[1]

    def to(self, device):
        return PagedInputs(self.q.to(device), self.k_cache.to(device), self.v_cache.to(device),
                           self.block_table.to(device), self.seq_lens.to(device),
                           self.block_size, self.scale, self.shared_groups)


def _cache(pool, H, bs, d, g, device, dtype):
    chunk = max(1, (1 << 26) // (H * bs * d))
    return _normal((pool, H, bs, d), g, device, dtype, 1.0, chunk)


def paged_uniform(num_seqs=64, H=32, d=128, block_size=16, pool=20000, len_lo=128, len_hi=4096,
                  seed=0, device="cpu", dtype=torch.bfloat16, max_blocks_per_seq=None, lens=None):
    """Paged decode workload with independent random placement.

    Draw order: seq_lens ~ U{len_lo..len_hi}; one randperm(pool), sliced
    consecutively into each sequence's ceil(L / block_size) blocks (so no
    physical block is used twice, within or across sequences); K cache;
    V cache; q.  Unused block-table entries are -1.  ``lens`` replaces the
    length draw with given lengths (edge-case tests).
    """
    g = _gen(seed, device)
    if lens is not None:
        seq_lens = torch.tensor(list(lens), dtype=torch.int64, device=device)
        num_seqs = len(lens)
    else:
        seq_lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g, device=device)
    perm = torch.randperm(pool, generator=g, device=device)
    seq_lens_c = seq_lens.cpu()
    perm_c = perm.cpu()
    mb = max_blocks_per_seq or -(-len_hi // block_size)
    table = torch.full((num_seqs, mb), -1, dtype=torch.int32)
    cur = 0
    for s in range(num_seqs):
        nb = -(-int(seq_lens_c[s]) // block_size)
        if cur + nb > pool:
            raise ValueError("pool too small for the drawn lengths")
        table[s, :nb] = perm_c[cur:cur + nb].to(torch.int32)
        cur += nb
    k_cache = _cache(pool, H, block_size, d, g, device, dtype)
    v_cache = _cache(pool, H, block_size, d, g, device, dtype)
    q = _normal((num_seqs, H, d), g, device, dtype)
    return PagedInputs(q, k_cache, v_cache, table.to(device), seq_lens.to(torch.int32).to(device),
                       block_size, 1.0 / math.sqrt(d))


def paged_shared_prefix(num_seqs=256, H=32, d=128, block_size=32, pool=20000, median=1024, sigma=1.0,
                        len_lo=1, len_hi=8192, group=8, prefix_tokens=512, seed=0, device="cpu",
                        dtype=torch.bfloat16):
    """Paged decode workload where groups of sequences share a common prefix.

    Draw order: z ~ N(0,1)[num_seqs] and seq_lens = clip(round(median *
    exp(sigma z)), len_lo, len_hi); one randperm(pool).  The permutation is
    sliced first into ``prefix_tokens / block_size`` prefix blocks for each
    group of ``group`` consecutive sequences, then into each sequence's own
    remaining blocks.  A sequence of length L uses the first
    ceil(min(L, prefix_tokens) / block_size) blocks of its group's prefix
    (shared, read-only: the same physical ids appear in several rows of the
    table), then its own blocks.  Then K cache, V cache, q.
    """
    g = _gen(seed, device)
    z = torch.randn(num_seqs, generator=g, device=device, dtype=torch.float64)
    seq_lens = torch.clamp(torch.round(median * torch.exp(sigma * z)), len_lo, len_hi).to(torch.int64)
    perm = torch.randperm(pool, generator=g, device=device).cpu()
    sl = seq_lens.cpu()
    pb = prefix_tokens // block_size
    n_groups = -(-num_seqs // group)
    mb = -(-len_hi // block_size)
    table = torch.full((num_seqs, mb), -1, dtype=torch.int32)
    cur = n_groups * pb
    if cur > pool:
        raise ValueError("pool too small for the shared prefixes")
    groups = []
    for gi in range(n_groups):
        prefix = perm[gi * pb:(gi + 1) * pb].to(torch.int32)
        members = list(range(gi * group, min(num_seqs, (gi + 1) * group)))
        groups.append(members)
        for s in members:
            L = int(sl[s])
            nb = -(-L // block_size)
            n_shared = min(nb, -(-min(L, prefix_tokens) // block_size))
            table[s, :n_shared] = prefix[:n_shared]
            n_own = nb - n_shared
            if cur + n_own > pool:
                raise ValueError("pool too small for the drawn lengths")
            table[s, n_shared:nb] = perm[cur:cur + n_own].to(torch.int32)
            cur += n_own
    k_cache = _cache(pool, H, block_size, d, g, device, dtype)
    v_cache = _cache(pool, H, block_size, d, g, device, dtype)
    q = _normal((num_seqs, H, d), g, device, dtype)
    return PagedInputs(q, k_cache, v_cache, table.to(device), seq_lens.to(torch.int32).to(device),
                       block_size, 1.0 / math.sqrt(d), groups)


@dataclass
class PagedPrefillInputs:
    q: torch.Tensor            # [total_q, Hq, d], sequence s owns rows cu_q[s] .. cu_q[s+1]-1
    k_cache: torch.Tensor      # [num_blocks, Hkv, block_size, d] (new tokens' keys included)
    v_cache: torch.Tensor
    block_table: torch.Tensor  # int32 [S, max_blocks_per_seq], unused entries -1
    seq_lens: torch.Tensor     # int32 [S], cached context + new tokens
    cu_q: torch.Tensor         # int32 [S + 1]
    block_size: int
    scale: float

    @property
    def num_seqs(self):
        return self.seq_lens.shape[0]

    @property
    def n_new(self):
        return (self.cu_q[1:] - self.cu_q[:-1]).cpu()

    def shuffled(self, seed=1):
        sh = shuffle_placement(PagedInputs(self.q, self.k_cache, self.v_cache, self.block_table, self.seq_lens,
                                           self.block_size, self.scale), seed=seed)
        return PagedPrefillInputs(self.q, sh.k_cache, sh.v_cache, sh.block_table, self.seq_lens, self.cu_q,
                                  self.block_size, self.scale)


def paged_prefill_inputs(ctx_lens, n_new, Hq=8, Hkv=8, d=128, block_size=16, pool=None, seed=0, device="cpu",
                         dtype=torch.bfloat16, max_blocks_per_seq=None):
    """Multi-token paged prefill inputs with given per-sequence cached context
    lengths and new-token counts (seq_lens = ctx + n).

    Draw order: one randperm(pool), sliced consecutively into each sequence's
    ceil(seq_len / block_size) blocks (no block used twice); K cache; V cache
    (N(0,1), every slot of the pool drawn, the new tokens' keys/values
    included); q [sum n, Hq, d].  Unused table entries are -1.
    """
    ctx_lens, n_new = [int(x) for x in ctx_lens], [int(x) for x in n_new]
    S = len(ctx_lens)
    lens = [c + n for c, n in zip(ctx_lens, n_new)]
    nbs = [-(-L // block_size) for L in lens]
    pool = pool or max(1, sum(nbs) + 2)
    g = _gen(seed, device)
    perm = torch.randperm(pool, generator=g, device=device).cpu()
    mb = max_blocks_per_seq or max(1, max(nbs) if nbs else 1)
    table = torch.full((S, mb), -1, dtype=torch.int32)
    cur = 0
    for s in range(S):
        if cur + nbs[s] > pool:
            raise ValueError("pool too small for the given lengths")
        table[s, :nbs[s]] = perm[cur:cur + nbs[s]].to(torch.int32)
        cur += nbs[s]
    k_cache = _cache(pool, Hkv, block_size, d, g, device, dtype)
    v_cache = _cache(pool, Hkv, block_size, d, g, device, dtype)
    cu = [0]
    for n in n_new:
        cu.append(cu[-1] + n)
    q = _normal((cu[-1], Hq, d), g, device, dtype, 1.0, max(1, (1 << 26) // (Hq * d)))
    return PagedPrefillInputs(q, k_cache, v_cache, table.to(device), torch.tensor(lens, dtype=torch.int32).to(device),
                              torch.tensor(cu, dtype=torch.int32).to(device), block_size, 1.0 / math.sqrt(d))


def paged_chunked_prefill(num_seqs=8, Hq=32, Hkv=8, d=128, block_size=16, pool=20000, chunk=2048, ctx_lo=0,
                          ctx_hi=6144, seed=0, device="cpu", dtype=torch.bfloat16):
    """Chunked-prefill workload: cached contexts ~ U{ctx_lo..ctx_hi} (drawn
    first, from the same generator seed + 1), then :func:`paged_prefill_inputs`
    with ``chunk`` new tokens per sequence."""
    gc = _gen(seed + 1, "cpu")
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (num_seqs,), generator=gc).tolist()
    mb = -(-(ctx_hi + chunk) // block_size)
    return paged_prefill_inputs(ctx, [chunk] * num_seqs, Hq, Hkv, d, block_size, pool, seed, device, dtype, mb)


def hadamard_signs(d=128, seed=0, device="cpu") -> torch.Tensor:
    """The random diagonal of incoherent processing: d int8 values, each +1
    or -1 with probability 1/2 (torch.randint from a CPU generator seeded
    ``seed``)."""
    g = _gen(seed, "cpu")
    return (torch.randint(0, 2, (d,), generator=g, dtype=torch.int8) * 2 - 1).to(device)


def shuffle_placement(inp: PagedInputs, seed=1, pool=None) -> PagedInputs:
    """Same logical data, new physical placement: every used physical block is
    moved to a new id by a random permutation of the pool, and the table is
    rewritten to match (shared blocks stay shared).  The logical K/V seen by
    each sequence is unchanged, so the attention result must be identical."""
    pool = pool or inp.num_blocks
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    perm = torch.randperm(pool, generator=g)
    dev = inp.k_cache.device
    perm_d = perm.to(dev)
    k_new = torch.empty_like(inp.k_cache)
    v_new = torch.empty_like(inp.v_cache)
    k_new[perm_d] = inp.k_cache
    v_new[perm_d] = inp.v_cache
    t = inp.block_table.cpu().to(torch.int64)
    t_new = torch.where(t >= 0, perm[t.clamp(min=0)], torch.full_like(t, -1)).to(torch.int32)
    return PagedInputs(inp.q, k_new, v_new, t_new.to(dev), inp.seq_lens, inp.block_size, inp.scale,
                       inp.shared_groups)


def unique_kv_bytes(inp: PagedInputs) -> int:
    """Bytes of distinct physical K/V rows that the decode must read: every
    (block, head, slot < tokens used in that block) counted once, even when
    several sequences share the block."""
    t = inp.block_table.cpu()
    sl = inp.seq_lens.cpu()
    used = {}
    bs = inp.block_size
    for s in range(t.shape[0]):
        L = int(sl[s])
        for lb in range(-(-L // bs)):
            phys = int(t[s, lb])
            n = min(bs, L - lb * bs)
            used[phys] = max(used.get(phys, 0), n)
    elem = inp.k_cache.element_size()
    return 2 * sum(used.values()) * inp.H * inp.d * elem


def logical_kv_bytes(inp: PagedInputs) -> int:
    """Bytes of K/V that the sequences attend over, shared blocks counted once
    per sequence: sum_s L_s * 2 * H * d * element size."""
    elem = inp.k_cache.element_size()
    return int(inp.seq_lens.cpu().to(torch.int64).sum()) * 2 * inp.H * inp.d * elem
