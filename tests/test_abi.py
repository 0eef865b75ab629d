"""C-ABI checks that need no GPU: the library loads, exports every function
include/attn.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import online_softmax_paged_b200 as osp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_0-9]+)\s*\([^;{]*\)\s*;", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(osp.lib_path()):
        from online_softmax_paged_b200 import build
        build.build()
    return osp.load()


def test_header_declares_expected_functions():
    assert _declared() == sorted(osp.EXPORTED_SYMBOLS)


def test_every_declared_symbol_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", osp.lib_path()], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(_declared()) <= exported
    # nothing else leaks: the kernels and helpers have hidden visibility
    assert not any(s.startswith("_ZN3osp") for s in exported)


def test_library_targets_sm100a_only():
    """Every source is compiled for sm_100a and nothing else (one -gencode
    pair, no PTX for other targets), by the build the library comes from."""
    from online_softmax_paged_b200 import build
    gencodes = [build.ARCH[i + 1] for i, a in enumerate(build.ARCH) if a == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"], build.ARCH


FAKE = ctypes.c_void_p(4096)  # 16-byte aligned, never dereferenced: checks fail first


def test_attn_fwd_rejects_on_host(lib):
    f = lib.attn_fwd
    ok_args = dict(B=1, H=2, N=8, d=128, causal=0, scale=0.125, dt=1)

    def call(**kw):
        a = {**ok_args, **kw}
        ptrs = [kw.get(p, FAKE) for p in ("Q", "K", "V", "O", "LSE")]
        return f(*ptrs, a["B"], a["H"], a["N"], a["d"], a["causal"], ctypes.c_float(a["scale"]), a["dt"], None, None)

    assert call(Q=None) == osp.ATTN_EINVAL
    assert call(N=0) == osp.ATTN_EINVAL
    assert call(B=0) == osp.ATTN_EINVAL
    assert call(scale=0.0) == osp.ATTN_EINVAL
    assert call(scale=float("nan")) == osp.ATTN_EINVAL
    assert call(dt=7) == osp.ATTN_EINVAL
    assert call(d=96) == osp.ATTN_EUNSUPPORTED
    assert call(d=256) == osp.ATTN_EUNSUPPORTED
    assert call(Q=ctypes.c_void_p(4097)) == osp.ATTN_EINVAL


def test_paged_decode_rejects_on_host(lib):
    f = lib.paged_attn_decode
    base = dict(block_size=16, S=2, H=4, d=128, nb=10, mb=4, scale=0.1, dt=1, ws=1 << 20)

    def call(**kw):
        a = {**base, **kw}
        p = [kw.get(n, FAKE) for n in ("q", "k", "v", "bt", "sl")]
        return f(*p, a["block_size"], kw.get("O", FAKE), kw.get("LSE", FAKE), a["S"], a["H"], a["d"], a["nb"],
                 a["mb"], ctypes.c_float(a["scale"]), a["dt"], kw.get("w", FAKE), a["ws"], None, None)

    assert call(q=None) == osp.ATTN_EINVAL
    assert call(dt=0) == osp.ATTN_EUNSUPPORTED
    assert call(d=64) == osp.ATTN_EUNSUPPORTED
    assert call(block_size=8) == osp.ATTN_EUNSUPPORTED
    assert call(block_size=64) == osp.ATTN_EUNSUPPORTED
    assert call(nb=0) == osp.ATTN_EINVAL
    assert call(scale=-1.0) == osp.ATTN_EINVAL
    assert call(ws=16) == osp.ATTN_EINVAL
    assert call(k=ctypes.c_void_p(4104)) == osp.ATTN_EINVAL
    assert call(S=0) == osp.ATTN_OK  # nothing to do, nothing launched


def test_workspace_size_and_split(lib):
    ws = osp.paged_attn_decode_workspace_size(64, 32, 128, 256, 16)
    st = osp.paged_attn_decode_split_tokens(64, 32, 128, 256, 16)
    assert st >= 256 and st % 32 == 0
    splits = -(-256 * 16 // st)
    assert ws >= 64 * 32 * splits * (128 + 1) * 4
    assert ws % 256 == 0
    assert osp.paged_attn_decode_workspace_size(64, 32, 64, 256, 16) == 0
    assert osp.paged_attn_decode_workspace_size(64, 0, 128, 256, 16) == 0
    # the split size is a function of the sizes only
    assert st == osp.paged_attn_decode_split_tokens(64, 32, 128, 256, 16)


def test_status_strings(lib):
    for s in range(5):
        assert osp.attn_status_str(s)
    assert osp.attn_status_str(99) == "unknown status"


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        osp.attn_fwd(x, x, x)


def test_gqa_workspace_size(lib):
    """Grouped workspace: groups of 1 and 2 need the multi-head size; groups
    of 4 and more at least that and room for the balanced schedule's partial
    rows (a bound of 1480 runs x up to 8 heads + one per query head, d + 1
    floats each),
    which dominates for few short sequences; invalid groupings give 0."""
    mha = osp.paged_attn_decode_workspace_size(64, 32, 128, 256, 16)
    for hkv in (32, 16):
        assert osp.paged_attn_decode_gqa_workspace_size(64, 32, hkv, 128, 256, 16) == mha
    for hkv in (8, 4, 1):
        assert osp.paged_attn_decode_gqa_workspace_size(64, 32, hkv, 128, 256, 16) >= mha
    small = osp.paged_attn_decode_gqa_workspace_size(1, 8, 1, 128, 4, 16)
    assert small > osp.paged_attn_decode_workspace_size(1, 8, 128, 4, 16)
    assert small >= (1480 * 8 + 8) * 129 * 4
    assert osp.paged_attn_decode_gqa_workspace_size(64, 32, 3, 128, 256, 16) == 0
    assert osp.paged_attn_decode_gqa_workspace_size(64, 32, 0, 128, 256, 16) == 0


C_CLIENT = r"""
#include <stdio.h>
#include "attn.h"

/* A plain C caller: no CUDA or PyTorch headers, only the library's. */
int main(void) {
    size_t ws = paged_attn_decode_workspace_size(64, 32, 128, 256, 16);
    size_t wg = paged_attn_decode_gqa_workspace_size(64, 32, 4, 128, 256, 16);
    int split = paged_attn_decode_split_tokens(64, 32, 128, 256, 16);
    /* host-side argument checks reject these before any CUDA call */
    attn_status s1 = attn_fwd(0, 0, 0, 0, 0, 1, 1, 1, 128, 0, 0.1f, ATTN_BF16, 0, 0);
    attn_status s2 = paged_attn_decode(0, 0, 0, 0, 0, 16, 0, 0, 1, 1, 128, 1, 1, 0.1f, ATTN_BF16, 0, 0, 0, 0);
    attn_status s3 = attn_selftest_wait_timeout(0, 0, 0);
    printf("%zu %zu %d %s %s %s\n", ws, wg, split, attn_status_str(s1), attn_status_str(s2), attn_status_str(s3));
    return (ws > 0 && wg >= ws && split > 0 && s1 == ATTN_EINVAL && s2 == ATTN_EINVAL && s3 == ATTN_EINVAL) ? 0 : 1;
}
"""


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    """The header is C99 (warnings as errors) and a C program links against
    the library with nothing but it; the host-only calls run without a GPU."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(osp.lib_path())
    libname = os.path.basename(osp.lib_path())
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                         str(src), "-o", str(exe), os.path.join(libdir, libname), "-Wl,-rpath," + libdir],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    fields = run.stdout.split()
    assert int(fields[0]) == osp.paged_attn_decode_workspace_size(64, 32, 128, 256, 16)
    # the library needs no PyTorch: its dynamic dependencies are system ones
    deps = subprocess.run(["ldd", osp.lib_path()], capture_output=True, text=True).stdout
    assert "torch" not in deps and "c10" not in deps, deps
