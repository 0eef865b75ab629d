"""GPU parity of the paged decode entry point against the fp64 oracle.

The oracle resolves every block table by explicit copy on the host; the
kernel gathers through the table on the device.  Small workloads are checked
in full (lengths 0, 1, 15, 16, 17, ..., max; block sizes 16 and 32); the two
full-size decode workloads on sampled sequences; physical placement shuffles
must give bit-identical output; bad tables and lengths set the device error
bits and zero the affected sequence.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import online_softmax_paged_b200 as osp
    osp.load()


def _osp():
    import online_softmax_paged_b200 as osp
    return osp


class DeviceCache:
    """Host view of a device cache that copies one physical block on access."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, i):
        return self.t[int(i)].float().cpu().numpy()


def _decode(p, err=None, **kw):
    O, LSE = _osp().paged_attn_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.block_size,
                                      scale=p.scale, err_flag=err, **kw)
    torch.cuda.synchronize()
    return O, LSE


def _oracle(p, seqs=None):
    return oracle.paged_decode(to64(p.q), DeviceCache(p.k_cache), DeviceCache(p.v_cache), p.block_table.cpu().numpy(),
                               p.seq_lens.cpu().numpy(), p.block_size, p.scale, seqs=seqs)


EDGE_LENS = [0, 1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257, 511, 513, 1000, 2048]


@pytest.mark.parametrize("bs", [16, 32])
def test_edge_lengths_full(bs):
    p = W.paged_uniform(H=32, d=128, block_size=bs, pool=600, len_hi=2048, seed=1, device="cuda", lens=EDGE_LENS)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _decode(p, err)
    assert int(err.item()) == 0
    O_ref, L_ref = _oracle(p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"edge lens bs={bs}")
    assert (O[0] == 0).all() and torch.isneginf(LSE[0]).all()  # seq_len 0


@pytest.mark.parametrize("bs", [16, 32])
def test_random_small_full(bs):
    p = W.paged_uniform(num_seqs=23, H=8, d=128, block_size=bs, pool=3000, len_lo=1, len_hi=3000, seed=2,
                        device="cuda")
    O, LSE = _decode(p)
    O_ref, L_ref = _oracle(p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"random bs={bs}")


def test_placement_shuffle_bit_identical_small():
    p = W.paged_uniform(num_seqs=11, H=4, d=128, block_size=16, pool=2000, len_lo=1, len_hi=3000, seed=3,
                        device="cuda")
    O1, L1 = _decode(p)
    for seed in (1, 2):
        O2, L2 = _decode(W.shuffle_placement(p, seed=seed))
        assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_decode_uniform_full_size():
    """64 sequences, H=32, d=128, bs=16, lengths U[128, 4096], pool 20000,
    seed 0: eight sampled sequences (shortest, longest and six others) in
    full against the oracle; all sequences for finiteness; a placement
    shuffle of the whole pool is bit-identical."""
    p = W.paged_uniform(device="cuda", seed=0, **W.DECODE_UNIFORM)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _decode(p, err)
    assert int(err.item()) == 0
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    sl = p.seq_lens.cpu().numpy()
    seqs = sorted({int(sl.argmin()), int(sl.argmax()), 0, 9, 21, 33, 47, 63})
    O_ref, L_ref = _oracle(p, seqs=seqs)
    check_close(O[seqs], LSE[seqs], O_ref[seqs], L_ref[seqs], torch.bfloat16, "decode uniform")
    O2, L2 = _decode(W.shuffle_placement(p, seed=11))
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


def test_decode_shared_prefix_full_size():
    """256 sequences, bs=32, log-normal lengths, 8-sequence groups sharing a
    512-token prefix, seed 0: two whole groups in full against the oracle."""
    p = W.paged_shared_prefix(device="cuda", seed=0, **W.DECODE_SHARED_PREFIX)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _decode(p, err)
    assert int(err.item()) == 0
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    seqs = p.shared_groups[0] + p.shared_groups[17]
    O_ref, L_ref = _oracle(p, seqs=seqs)
    check_close(O[seqs], LSE[seqs], O_ref[seqs], L_ref[seqs], torch.bfloat16, "decode shared prefix")


def test_bad_block_table_entry_flags_and_zeroes():
    osp = _osp()
    p = W.paged_uniform(num_seqs=6, H=4, d=128, block_size=16, pool=900, len_lo=100, len_hi=1500, seed=4,
                        device="cuda")
    t = p.block_table.clone()
    t[2, 3] = p.num_blocks + 5
    t[4, 0] = -7
    bad = W.PagedInputs(p.q, p.k_cache, p.v_cache, t, p.seq_lens, p.block_size, p.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _decode(bad, err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_BLOCK_TABLE
    for s in (2, 4):
        assert (O[s] == 0).all() and torch.isneginf(LSE[s]).all()
    good = [0, 1, 3, 5]
    O_ref, L_ref = _oracle(p, seqs=good)
    check_close(O[good], LSE[good], O_ref[good], L_ref[good], torch.bfloat16, "good rows beside bad ones")


def test_bad_seq_len_flags_and_zeroes():
    osp = _osp()
    p = W.paged_uniform(num_seqs=4, H=4, d=128, block_size=16, pool=500, len_lo=10, len_hi=400, seed=5,
                        device="cuda")
    sl = p.seq_lens.clone()
    sl[1] = p.max_blocks_per_seq * 16 + 1
    sl[3] = -2
    bad = W.PagedInputs(p.q, p.k_cache, p.v_cache, p.block_table, sl, p.block_size, p.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _decode(bad, err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_SEQ_LEN
    for s in (1, 3):
        assert (O[s] == 0).all() and torch.isneginf(LSE[s]).all()
    O_ref, L_ref = _oracle(p, seqs=[0, 2])
    check_close(O[[0, 2]], LSE[[0, 2]], O_ref[[0, 2]], L_ref[[0, 2]], torch.bfloat16, "good rows")


def test_workspace_too_small_rejected():
    osp = _osp()
    p = W.paged_uniform(num_seqs=3, H=4, d=128, block_size=16, pool=300, len_lo=10, len_hi=400, seed=6,
                        device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(osp.AttnError):
        _decode(p, workspace=ws)


def test_decode_equals_dense_last_row():
    """Paging changes storage, not the math: with an identity table the decode
    of the last token equals the dense causal prefill's last row (both within
    tolerance of the same oracle value)."""
    osp = _osp()
    H, d, bs, L = 4, 128, 16, 700
    nb = -(-L // bs)
    dense = W.dense_inputs(1, H, nb * bs, d, dtype=torch.bfloat16, seed=9, device="cuda", causal=True)
    kc = dense["K"][0].view(H, nb, bs, d).permute(1, 0, 2, 3).contiguous()
    vc = dense["V"][0].view(H, nb, bs, d).permute(1, 0, 2, 3).contiguous()
    q = dense["Q"][0, :, L - 1].contiguous().view(1, H, d)
    table = torch.arange(nb, dtype=torch.int32, device="cuda").view(1, nb)
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    O, LSE = osp.paged_attn_decode(q, kc, vc, table, sl, bs)
    Od, Ld = osp.attn_fwd(dense["Q"][:, :, :L].contiguous(), dense["K"][:, :, :L].contiguous(),
                          dense["V"][:, :, :L].contiguous(), causal=True)
    torch.cuda.synchronize()
    assert (O[0].float() - Od[0, :, L - 1].float()).abs().max().item() <= 2e-2
    assert (LSE[0] - Ld[0, :, L - 1]).abs().max().item() <= 1e-3


@pytest.mark.parametrize("G,bs", [(2, 16), (4, 32), (8, 16), (4, 16), (8, 32), (2, 32)])
def test_gqa_decode_full(G, bs):
    """Grouped-query decode: H_q = 32 query heads over 32 / G key/value heads,
    lengths 0..3000 (edge lengths included), against the grouped oracle."""
    osp = _osp()
    Hkv = 32 // G
    lens = [0, 1, 17, 255, 256, 257, 1000, 3000, 2048, 5]
    p = W.paged_uniform(H=Hkv, d=128, block_size=bs, pool=1200, len_hi=3000, seed=12 + G, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(40 + G)
    q = torch.randn((len(lens), 32, 128), generator=g, device="cuda").to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = osp.paged_attn_decode_gqa(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, bs, scale=p.scale,
                                       err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    O_ref, L_ref = oracle.paged_decode(to64(q), DeviceCache(p.k_cache), DeviceCache(p.v_cache),
                                       p.block_table.cpu().numpy(), p.seq_lens.cpu().numpy(), bs, p.scale)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"gqa G={G} bs={bs}")
    # placement shuffle: bit-identical
    p2 = W.shuffle_placement(p, seed=3)
    O2, L2 = osp.paged_attn_decode_gqa(q, p2.k_cache, p2.v_cache, p2.block_table, p2.seq_lens, bs, scale=p.scale)
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


def test_gqa_group_one_is_multi_head():
    osp = _osp()
    p = W.paged_uniform(num_seqs=9, H=8, d=128, block_size=16, pool=900, len_lo=1, len_hi=1500, seed=30,
                        device="cuda")
    O1, L1 = _decode(p)
    O2, L2 = osp.paged_attn_decode_gqa(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, 16, scale=p.scale)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_gqa_decode_bad_group_rejected():
    osp = _osp()
    p = W.paged_uniform(num_seqs=2, H=4, d=128, block_size=16, pool=100, len_lo=1, len_hi=100, seed=31,
                        device="cuda")
    q = torch.zeros((2, 12, 128), dtype=torch.bfloat16, device="cuda")  # group of 3
    with pytest.raises(osp.AttnError):
        osp.paged_attn_decode_gqa(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, 16)


@pytest.mark.parametrize("G", [1, 4, 8])
def test_nan_in_unused_cache_slots_does_not_leak(G):
    """Every cache slot no sequence uses (tails of last blocks, unused blocks)
    set to NaN: the output equals the clean run bit for bit."""
    osp = _osp()
    Hkv = 32 // G
    lens = [1, 17, 255, 300, 1000, 33, 2047]
    p = W.paged_uniform(H=Hkv, d=128, block_size=32, pool=400, len_hi=2048, seed=50 + G, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(60 + G)
    q = torch.randn((len(lens), 32, 128), generator=g, device="cuda").to(torch.bfloat16)
    O1, L1 = osp.paged_attn_decode_gqa(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, 32, scale=p.scale)
    live = torch.zeros(p.k_cache.shape[0], 32, dtype=torch.bool)
    t, sl = p.block_table.cpu(), p.seq_lens.cpu()
    for s in range(t.shape[0]):
        L = int(sl[s])
        for lb in range(-(-L // 32)):
            live[int(t[s, lb]), :min(32, L - lb * 32)] = True
    dead = (~live).to("cuda")[:, None, :, None]
    kc = p.k_cache.clone().masked_fill_(dead, float("nan"))
    vc = p.v_cache.clone().masked_fill_(dead, float("nan"))
    O2, L2 = osp.paged_attn_decode_gqa(q, kc, vc, p.block_table, p.seq_lens, 32, scale=p.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(O2.float()).all()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


@pytest.mark.parametrize("Hq,Hkv,bs", [(32, 1, 16), (32, 2, 32), (64, 4, 16)])
def test_mqa_large_groups_full(Hq, Hkv, bs):
    """Groups above 8 (multi-query attention at H_kv = 1): 32 or 64 query
    heads over 1, 2 or 4 key/value heads against the grouped oracle, edge
    lengths included; a placement shuffle is bit-identical."""
    osp = _osp()
    lens = [0, 1, 17, 255, 256, 257, 1000, 3000, 33]
    p = W.paged_uniform(H=Hkv, d=128, block_size=bs, pool=1200, len_hi=3000, seed=70 + Hq + Hkv, device="cuda",
                        lens=lens)
    g = torch.Generator(device="cuda").manual_seed(80 + Hkv)
    q = torch.randn((len(lens), Hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = osp.paged_attn_decode_gqa(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, bs, scale=p.scale,
                                       err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    O_ref, L_ref = oracle.paged_decode(to64(q), DeviceCache(p.k_cache), DeviceCache(p.v_cache),
                                       p.block_table.cpu().numpy(), p.seq_lens.cpu().numpy(), bs, p.scale)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"mqa Hq={Hq} Hkv={Hkv} bs={bs}")
    p2 = W.shuffle_placement(p, seed=5)
    O2, L2 = osp.paged_attn_decode_gqa(q, p2.k_cache, p2.v_cache, p2.block_table, p2.seq_lens, bs, scale=p.scale)
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


def _gqa(q, p, err=None):
    O, LSE = _osp().paged_attn_decode_gqa(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.block_size,
                                          scale=p.scale, err_flag=err)
    torch.cuda.synchronize()
    return O, LSE


def _gqa_oracle(q, p, seqs=None):
    return oracle.paged_decode(to64(q), DeviceCache(p.k_cache), DeviceCache(p.v_cache), p.block_table.cpu().numpy(),
                               p.seq_lens.cpu().numpy(), p.block_size, p.scale, seqs=seqs)


@pytest.mark.parametrize("Hq,bs", [(8, 16), (4, 32)])
def test_gqa_long_row_many_segments(Hq, bs):
    """Groups of 4 and 8 run on a balanced schedule that cuts the (sequence,
    key/value head) rows into equal runs of tiles.  Few tiles in all give the
    shortest run (128 keys), so a 20000-token row is cut into more than 128
    segments (the merge kernel's batches of 32 partials) beside short rows;
    a placement shuffle is bit-identical."""
    lens = [20000, 1, 16, 17, 700]
    p = W.paged_uniform(H=1, d=128, block_size=bs, pool=1400, len_hi=20000, seed=90 + Hq, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(91 + Hq)
    q = torch.randn((len(lens), Hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _gqa(q, p, err)
    assert int(err.item()) == 0
    O_ref, L_ref = _gqa_oracle(q, p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"long row Hq={Hq} bs={bs}")
    p2 = W.shuffle_placement(p, seed=7)
    O2, L2 = _gqa(q, p2)
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


def test_gqa_odd_runs_cut_blocks():
    """64 sequences of 0..850 tokens, 8 key/value heads, G = 4, 32-token
    blocks: 12776 tiles over 1184 workers give runs of 11 tiles, so runs start and end in
    the middle of cache blocks and rows; against the oracle, and a placement
    shuffle is bit-identical."""
    lens = np.random.default_rng(95).integers(0, 851, 64).tolist()  # lengths fixed on the host
    p = W.paged_uniform(H=8, d=128, block_size=32, pool=1700, len_hi=850, seed=93, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(94)
    q = torch.randn((64, 32, 128), generator=g, device="cuda").to(torch.bfloat16)
    tiles = int(sum(-(-int(L) // 16) for L in lens)) * 8
    assert -(-tiles // 1184) % 2 == 1, tiles  # an odd run length
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _gqa(q, p, err)
    assert int(err.item()) == 0
    O_ref, L_ref = _gqa_oracle(q, p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "odd runs bs=32")
    p2 = W.shuffle_placement(p, seed=8)
    O2, L2 = _gqa(q, p2)
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


@pytest.mark.parametrize("G", [4, 8])
def test_gqa_bad_block_table_entry_in_cut_row(G):
    """A bad block id deep inside a long row that spans several runs: the
    error bit is set, that sequence is zeroed (O = 0, LSE = -inf) for every
    query head, the other sequences still match the oracle."""
    osp = _osp()
    Hkv = 32 // G
    lens = [3000, 5000, 40, 2500]
    p = W.paged_uniform(H=Hkv, d=128, block_size=16, pool=700, len_hi=5000, seed=95 + G, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(96 + G)
    q = torch.randn((len(lens), 32, 128), generator=g, device="cuda").to(torch.bfloat16)
    t = p.block_table.clone()
    t[1, 200] = p.num_blocks + 3
    bad = W.PagedInputs(q, p.k_cache, p.v_cache, t, p.seq_lens, p.block_size, p.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _gqa(q, bad, err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_BLOCK_TABLE
    assert (O[1] == 0).all() and torch.isneginf(LSE[1]).all()
    good = [0, 2, 3]
    O_ref, L_ref = _gqa_oracle(q, p, seqs=good)
    check_close(O[good], LSE[good], O_ref[good], L_ref[good], torch.bfloat16, f"G={G} good rows beside a bad one")


@pytest.mark.parametrize("G", [4, 8])
def test_gqa_bad_seq_len_flags_and_zeroes(G):
    """Grouped decode plans inside its own kernel: an invalid length (too long,
    negative) still sets the error bit and zeroes that sequence, an empty one
    is O = 0 / LSE = -inf without the bit, the others match the oracle."""
    osp = _osp()
    Hkv = 32 // G
    lens = [300, 700, 0, 1500, 64]
    p = W.paged_uniform(H=Hkv, d=128, block_size=16, pool=300, len_hi=1500, seed=97 + G, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(98 + G)
    q = torch.randn((len(lens), 32, 128), generator=g, device="cuda").to(torch.bfloat16)
    sl = p.seq_lens.clone()
    sl[1] = p.block_table.shape[1] * 16 + 1
    sl[4] = -3
    bad = W.PagedInputs(q, p.k_cache, p.v_cache, p.block_table, sl, p.block_size, p.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _gqa(q, bad, err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_SEQ_LEN
    for s in (1, 2, 4):
        assert (O[s] == 0).all() and torch.isneginf(LSE[s]).all()
    good = [0, 3]
    O_ref, L_ref = _gqa_oracle(q, p, seqs=good)
    check_close(O[good], LSE[good], O_ref[good], L_ref[good], torch.bfloat16, f"G={G} good rows beside bad lengths")


@pytest.mark.parametrize("G", [4, 8])
def test_gqa_many_sequences_plan_kernel(G):
    """Above 4096 sequences the grouped kernel takes its offsets from the
    plan kernel (global memory) instead of planning in shared memory: 4100
    short sequences (0..40 tokens, some empty), against the oracle, and a
    placement shuffle is bit-identical."""
    lens = np.random.default_rng(120 + G).integers(0, 41, 4100).tolist()
    p = W.paged_uniform(H=8 // G, d=128, block_size=16, pool=12400, len_hi=40, seed=121 + G, device="cuda", lens=lens)
    g = torch.Generator(device="cuda").manual_seed(122 + G)
    q = torch.randn((len(lens), 8, 128), generator=g, device="cuda").to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _gqa(q, p, err)
    assert int(err.item()) == 0
    O_ref, L_ref = _gqa_oracle(q, p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"4100 sequences G={G}")
    p2 = W.shuffle_placement(p, seed=9)
    O2, L2 = _gqa(q, p2)
    assert torch.equal(O, O2) and torch.equal(LSE, L2)
