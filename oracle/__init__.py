"""Oracle for exact attention forward (dense prefill and paged decode).

TEST INFRASTRUCTURE ONLY: a plain, slow, fp64 CPU implementation used to
check the CUDA library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` import it.  The library package
never imports it and it imports nothing from the library.

Parity pins (what each function is checked against, other than itself) live
in ``tests/test_oracle.py``; every function here is pinned.
"""
from .attention import (  # noqa: F401
    NEG_INF,
    attention_dense,
    attention_flops,
    attention_head,
    attention_online_tiled,
    block_copy,
    cow_plan,
    gather_paged,
    kv_append,
    merge_partials,
    paged_decode,
    paged_prefill,
    scores,
    softmax_probs,
)
from .brute import brute_attention, brute_paged_decode, build_brute  # noqa: F401
from . import fp8  # noqa: F401,E402  (e4m3 block quantisation with incoherent processing)
