"""Python binding of the sm_100a exact-attention library (``include/attn.h``).

Argument marshalling only: every step of attention runs in the CUDA kernels
of ``libattn_sm100.so``.  PyTorch supplies device memory and the stream.
There is no fallback: if the library is missing or a tensor is not on a CUDA
device the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "AttnError", "attn_fwd", "paged_attn_decode", "paged_attn_decode_workspace_size",
    "paged_attn_decode_split_tokens", "paged_attn_decode_noalloc", "attn_read_error", "attn_status_str", "lib_path", "load",
    "ATTN_DEVERR_BLOCK_TABLE", "ATTN_DEVERR_SEQ_LEN", "ATTN_DEVERR_TIMEOUT", "ATTN_DEVERR_INDEX",
    "EXPORTED_SYMBOLS", "paged_kv_append", "paged_block_copy", "paged_attn_decode_gqa", "paged_attn_prefill",
    "attn_quantize_fp8", "attn_fwd_fp8", "paged_attn_decode_gqa_workspace_size", "attn_selftest_wait_timeout",
    "attn_selftest_exp2_poly", "paged_cow_plan",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libattn_sm100.so")

ATTN_OK, ATTN_EINVAL, ATTN_EUNSUPPORTED, ATTN_ECUDA, ATTN_EDEVICE, ATTN_ENOBLOCKS = range(6)
ATTN_F32, ATTN_BF16 = 0, 1
ATTN_DEVERR_BLOCK_TABLE, ATTN_DEVERR_SEQ_LEN, ATTN_DEVERR_TIMEOUT, ATTN_DEVERR_INDEX = 1, 2, 4, 8

# every function include/attn.h declares
EXPORTED_SYMBOLS = ("attn_fwd", "paged_attn_decode_workspace_size", "paged_attn_decode_gqa_workspace_size",
                    "paged_attn_decode_split_tokens",
                    "paged_attn_decode", "paged_attn_decode_gqa", "paged_attn_decode_noalloc", "paged_attn_prefill",
                    "attn_quantize_fp8", "attn_fwd_fp8",
                    "paged_kv_append",
                    "paged_block_copy", "paged_cow_plan",
                    "attn_read_error", "attn_status_str", "attn_selftest_wait_timeout", "attn_selftest_exp2_poly")

# size of the fixed scratch array paged_attn_decode_noalloc uses (attn.h)
ATTN_NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {attn_status_str(status)} (status {status})")


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m online_softmax_paged_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32p, fp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p
    c_int, c_float, c_size = ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, fp, c_int, c_int, c_int, c_int, c_int, c_float, c_int, vp, vp]
    lib.attn_fwd.restype = c_int
    lib.paged_attn_decode_workspace_size.argtypes = [c_int] * 5
    lib.paged_attn_decode_workspace_size.restype = c_size
    lib.paged_attn_decode_gqa_workspace_size.argtypes = [c_int] * 6
    lib.paged_attn_decode_gqa_workspace_size.restype = c_size
    lib.paged_attn_decode_split_tokens.argtypes = [c_int] * 5
    lib.paged_attn_decode_split_tokens.restype = c_int
    lib.paged_attn_decode.argtypes = [vp, vp, vp, vp, vp, c_int, vp, fp, c_int, c_int, c_int, c_int, c_int,
                                      c_float, c_int, vp, c_size, vp, vp]
    lib.paged_attn_decode.restype = c_int
    lib.paged_attn_decode_gqa.argtypes = [vp, vp, vp, vp, vp, c_int, vp, fp, c_int, c_int, c_int, c_int, c_int,
                                          c_int, c_float, c_int, vp, c_size, vp, vp]
    lib.paged_attn_decode_gqa.restype = c_int
    lib.paged_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, c_int, vp, fp, c_int, c_int, c_int, c_int, c_int,
                                              c_float, c_int, vp, vp]
    lib.paged_attn_decode_noalloc.restype = c_int
    lib.attn_quantize_fp8.argtypes = [vp, vp, vp, c_int, c_int, c_int, vp, vp]
    lib.attn_quantize_fp8.restype = c_int
    lib.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_float, vp, vp]
    lib.attn_fwd_fp8.restype = c_int
    lib.paged_attn_prefill.argtypes = [vp, vp, vp, vp, vp, vp, c_int, vp, fp, c_int, c_int, c_int, c_int, c_int,
                                       c_int, c_int, c_int, c_float, c_int, vp, vp]
    lib.paged_attn_prefill.restype = c_int
    lib.paged_kv_append.argtypes = [vp, vp, vp, vp, c_int, vp, c_int, c_int, vp, vp, c_int, c_int, c_int, c_int,
                                    c_int, vp, vp]
    lib.paged_kv_append.restype = c_int
    lib.paged_block_copy.argtypes = [vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, vp, vp]
    lib.paged_block_copy.restype = c_int
    lib.paged_cow_plan.argtypes = [vp, c_int, c_int, vp, c_int, vp, vp, vp, vp, c_int, vp, vp, vp]
    lib.paged_cow_plan.restype = c_int
    lib.attn_read_error.argtypes = [vp, i32p, vp]
    lib.attn_read_error.restype = c_int
    lib.attn_selftest_wait_timeout.argtypes = [vp, vp, vp]
    lib.attn_selftest_wait_timeout.restype = c_int
    lib.attn_selftest_exp2_poly.argtypes = [vp, vp, c_int, vp]
    lib.attn_selftest_exp2_poly.restype = c_int
    lib.attn_status_str.argtypes = [c_int]
    lib.attn_status_str.restype = ctypes.c_char_p
    _lib = lib
    return lib


def attn_status_str(status: int) -> str:
    return load().attn_status_str(int(status)).decode()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _check_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be on a CUDA device (the library has no CPU path)")


def _check_device(dev, *ts):
    """Every given tensor must be on ``dev``: the library launches on the
    device that holds the inputs and reads every pointer there."""
    for t in ts:
        if t is not None and t.device != dev:
            raise ValueError(f"all tensors must be on {dev} (got one on {t.device})")


def _check_tensor(t, shape, dtype, name):
    """``t`` (when given) must be a contiguous ``dtype`` tensor of ``shape``:
    the kernels index it by the sizes passed, so anything smaller would be
    read or written past its end."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} "
                         f"(got {t.dtype} {tuple(t.shape)}{'' if t.is_contiguous() else ', not contiguous'})")


def _check_err_flag(err_flag):
    if err_flag is not None and (err_flag.dtype != torch.int32 or err_flag.numel() < 1):
        raise ValueError("err_flag must be an int32 tensor with at least one element")


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return ATTN_BF16
    if dt == torch.float32:
        return ATTN_F32
    raise ValueError(f"unsupported dtype {dt}")


def attn_fwd(Q, K, V, O=None, LSE=None, causal=False, scale=None, err_flag=None, stream=None):
    """Dense attention forward.  Q, K, V: [B, H, N, d] contiguous CUDA tensors of
    one dtype (bf16 or fp32).  Returns (O, LSE); O and LSE are allocated when
    not given.  See ``attn_fwd`` in include/attn.h for the contract."""
    _check_cuda(Q, K, V, O, LSE, err_flag)
    B, H, N, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape or K.dtype != Q.dtype or V.dtype != Q.dtype:
        raise ValueError("Q, K, V must share shape and dtype")
    if not (Q.is_contiguous() and K.is_contiguous() and V.is_contiguous()):
        raise ValueError("Q, K, V must be contiguous")
    _check_device(Q.device, K, V, O, LSE, err_flag)
    _check_tensor(O, Q.shape, Q.dtype, "O")
    _check_tensor(LSE, (B, H, N), torch.float32, "LSE")
    _check_err_flag(err_flag)
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(Q.device):
        st = load().attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, N, d, int(bool(causal)),
                             float(scale), _dtype_code(Q.dtype), _ptr(err_flag), _stream(stream, Q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")
    return O, LSE


def attn_quantize_fp8(x, signs=None, codes=None, scales=None, stream=None):
    """Block-quantise bf16 rows x [..., N, d] (d = 128, contiguous) to e4m3
    with one scale per 128 rows of each leading index; ``signs`` (d int8
    values of +-1) turns on incoherent processing.  Returns (codes uint8,
    same shape as x, viewable as torch.float8_e4m3fn; scales fp32
    [..., ceil(N / 128)]).  See include/attn.h."""
    _check_cuda(x, signs, codes, scales)
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be contiguous bf16")
    *lead, N, d = x.shape
    BH = int(math.prod(lead)) if lead else 1
    nblk = -(-N // 128)
    _check_device(x.device, signs, codes, scales)
    _check_tensor(codes, x.shape, torch.uint8, "codes")
    _check_tensor(scales, tuple(lead) + (nblk,), torch.float32, "scales")
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(tuple(lead) + (nblk,), dtype=torch.float32, device=x.device)
    if signs is not None and (signs.dtype != torch.int8 or signs.numel() != d or not signs.is_contiguous()):
        raise ValueError("signs must be d contiguous int8 values")
    with torch.cuda.device(x.device):
        st = load().attn_quantize_fp8(_ptr(x), _ptr(codes), _ptr(scales), BH, N, d, _ptr(signs),
                                      _stream(stream, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_quantize_fp8")
    return codes, scales


def attn_fwd_fp8(q8, q_scale, k8, k_scale, V, O=None, LSE=None, causal=False, scale=None, err_flag=None,
                 stream=None):
    """FP8 prefill: e4m3 Q and K [B, H, N, d] (uint8 or float8_e4m3fn) with
    their block scales [B, H, ceil(N / 128)] from attn_quantize_fp8, bf16 V
    [B, H, N, d].  Returns (O bf16, LSE fp32).  See include/attn.h."""
    _check_cuda(q8, q_scale, k8, k_scale, V, O, LSE, err_flag)
    B, H, N, d = V.shape
    if q8.shape != V.shape or k8.shape != V.shape or q8.element_size() != 1 or k8.element_size() != 1:
        raise ValueError("q8 and k8 must be one-byte tensors of V's shape")
    if V.dtype != torch.bfloat16:
        raise ValueError("V must be bf16")
    for t in (q8, q_scale, k8, k_scale, V):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    nblk = -(-N // 128)
    _check_tensor(q_scale, (B, H, nblk), torch.float32, "q_scale")
    _check_tensor(k_scale, (B, H, nblk), torch.float32, "k_scale")
    _check_device(V.device, q8, q_scale, k8, k_scale, O, LSE, err_flag)
    _check_tensor(O, V.shape, torch.bfloat16, "O")
    _check_tensor(LSE, (B, H, N), torch.float32, "LSE")
    _check_err_flag(err_flag)
    if O is None:
        O = torch.empty_like(V)
    if LSE is None:
        LSE = torch.empty((B, H, N), dtype=torch.float32, device=V.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(V.device):
        st = load().attn_fwd_fp8(_ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(V), _ptr(O), _ptr(LSE), B,
                                 H, N, d, int(bool(causal)), float(scale), _ptr(err_flag), _stream(stream, V.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return O, LSE


def _check_decode_args(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE, err_flag, grouped):
    """Shapes, dtypes, layout and device of a paged decode call's tensors.
    Returns (S, H_q, H_kv, d, num_blocks, max_blocks_per_seq)."""
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [S, H, d] and the caches [num_blocks, H_kv, block_size, d]")
    S, Hq, d = q.shape
    nb, Hkv, bs, dk = k_cache.shape
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    if k_cache.shape != v_cache.shape or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype or \
            bs != block_size or dk != d or (not grouped and Hkv != Hq):
        raise ValueError("caches must be [num_blocks, H, block_size, d] of q's dtype"
                         + (" (H = H_kv)" if grouped else ""))
    if block_table.dim() != 2 or block_table.shape[0] != S:
        raise ValueError(f"block_table must be [S, max_blocks_per_seq] with S = {S}")
    if tuple(seq_lens.shape) != (S,):
        raise ValueError(f"seq_lens must hold S = {S} lengths")
    for t in (q, k_cache, v_cache, block_table, seq_lens):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    _check_device(q.device, k_cache, v_cache, block_table, seq_lens, O, LSE, err_flag)
    _check_tensor(O, q.shape, q.dtype, "O")
    _check_tensor(LSE, (S, Hq), torch.float32, "LSE")
    _check_err_flag(err_flag)
    return S, Hq, Hkv, d, nb, block_table.shape[1]


def _check_workspace(workspace, dev):
    if workspace is None:
        return
    _check_device(dev, workspace)
    if not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")


def paged_attn_decode_workspace_size(num_seqs, H, d, max_blocks_per_seq, block_size) -> int:
    return int(load().paged_attn_decode_workspace_size(num_seqs, H, d, max_blocks_per_seq, block_size))


def paged_attn_decode_gqa_workspace_size(num_seqs, H_q, H_kv, d, max_blocks_per_seq, block_size) -> int:
    return int(load().paged_attn_decode_gqa_workspace_size(int(num_seqs), int(H_q), int(H_kv), int(d),
                                                           int(max_blocks_per_seq), int(block_size)))


def paged_attn_decode_split_tokens(num_seqs, H, d, max_blocks_per_seq, block_size) -> int:
    return int(load().paged_attn_decode_split_tokens(num_seqs, H, d, max_blocks_per_seq, block_size))


def paged_attn_decode(q, k_cache, v_cache, block_table, seq_lens, block_size, O=None, LSE=None, scale=None,
                      workspace=None, err_flag=None, stream=None):
    """Paged decode.  q [S, H, d] bf16; caches [num_blocks, H, block_size, d]
    bf16; block_table int32 [S, max_blocks_per_seq]; seq_lens int32 [S].
    Returns (O, LSE).  ``workspace`` (uint8 CUDA tensor) is allocated when
    not given.  See ``paged_attn_decode`` in include/attn.h."""
    _check_cuda(q, k_cache, v_cache, block_table, seq_lens, O, LSE, workspace, err_flag)
    S, H, _, d, num_blocks, mb = _check_decode_args(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE,
                                                    err_flag, grouped=False)
    _check_workspace(workspace, q.device)
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((S, H), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        if workspace is None:  # (a given workspace is checked against the need by the library)
            need = paged_attn_decode_workspace_size(S, H, d, mb, block_size)
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        st = load().paged_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                      int(block_size), _ptr(O), _ptr(LSE), S, H, d, num_blocks, mb, float(scale),
                                      _dtype_code(q.dtype), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(err_flag),
                                      _stream(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_attn_decode")
    return O, LSE


def paged_attn_decode_gqa(q, k_cache, v_cache, block_table, seq_lens, block_size, O=None, LSE=None, scale=None,
                          workspace=None, err_flag=None, stream=None):
    """Grouped-query paged decode: q [S, H_q, d], caches [num_blocks, H_kv,
    block_size, d] with H_q / H_kv in {1, 2, 4} or a multiple of 8 (H_kv = 1:
    multi-query attention).  See include/attn.h."""
    _check_cuda(q, k_cache, v_cache, block_table, seq_lens, O, LSE, workspace, err_flag)
    S, Hq, Hkv, d, nb, mb = _check_decode_args(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE,
                                               err_flag, grouped=True)
    _check_workspace(workspace, q.device)
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        if workspace is None:  # (a given workspace is checked against the need by the library)
            need = paged_attn_decode_gqa_workspace_size(S, Hq, Hkv, d, mb, block_size)
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        st = load().paged_attn_decode_gqa(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                          _ptr(seq_lens), int(block_size), _ptr(O), _ptr(LSE), S, Hq, Hkv, d, nb, mb,
                                          float(scale), _dtype_code(q.dtype), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _ptr(err_flag),
                                          _stream(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_attn_decode_gqa")
    return O, LSE


def paged_attn_prefill(q, k_cache, v_cache, block_table, seq_lens, cu_q, block_size, max_q_per_seq=None, O=None,
                       LSE=None, scale=None, err_flag=None, stream=None):
    """Multi-token paged prefill: q [total_q, H_q, d] bf16 packed by cu_q
    (int32 [S + 1]); caches [num_blocks, H_kv, block_size, d] already holding
    the new tokens' keys/values; seq_lens counts them.  ``max_q_per_seq`` is
    read from cu_q (one device-to-host copy) when not given.  See
    include/attn.h."""
    _check_cuda(q, k_cache, v_cache, block_table, seq_lens, cu_q, O, LSE, err_flag)
    T, Hq, d = q.shape
    nb, Hkv, bs, dk = k_cache.shape
    S = seq_lens.shape[0]
    for t in (block_table, seq_lens, cu_q):
        if t.dtype != torch.int32:
            raise ValueError("block_table, seq_lens and cu_q must be int32")
    if cu_q.shape != (S + 1,) or block_table.shape[0] != S:
        raise ValueError("cu_q must be [S + 1] and block_table [S, max_blocks]")
    if k_cache.shape != v_cache.shape or bs != block_size or dk != d:
        raise ValueError("caches must be [num_blocks, H_kv, block_size, d]")
    if block_table.dim() != 2 or tuple(seq_lens.shape) != (S,):
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("caches must have q's dtype")
    for t in (q, k_cache, v_cache, block_table, seq_lens, cu_q):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    _check_device(q.device, k_cache, v_cache, block_table, seq_lens, cu_q, O, LSE, err_flag)
    _check_tensor(O, q.shape, q.dtype, "O")
    _check_tensor(LSE, (T, Hq), torch.float32, "LSE")
    _check_err_flag(err_flag)
    if max_q_per_seq is None:
        max_q_per_seq = int((cu_q[1:] - cu_q[:-1]).max().item()) if S > 0 else 0
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        st = load().paged_attn_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                       _ptr(cu_q), int(block_size), _ptr(O), _ptr(LSE), S, T, int(max_q_per_seq),
                                       Hq, Hkv, d, nb, block_table.shape[1], float(scale), _dtype_code(q.dtype),
                                       _ptr(err_flag), _stream(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_attn_prefill")
    return O, LSE


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_table, seq_lens, block_size, O=None, LSE=None,
                              scale=None, err_flag=None, stream=None):
    """Paged decode that passes no workspace: the library uses its own fixed
    scratch array (ATTN_NOALLOC_SCRATCH_BYTES), for callers that cannot
    allocate device memory.  Calls that may overlap on the GPU share that
    scratch and race; keep them on one stream.  The first call on a device
    looks up the scratch address, so make it before any graph capture.
    O and LSE are allocated here when not given (pass them to allocate
    nothing).  Raises AttnError (ATTN_EUNSUPPORTED) when the sizes need more
    scratch than the array holds."""
    _check_cuda(q, k_cache, v_cache, block_table, seq_lens, O, LSE, err_flag)
    S, H, _, d, nb, mb = _check_decode_args(q, k_cache, v_cache, block_table, seq_lens, block_size, O, LSE,
                                            err_flag, grouped=False)
    if O is None:
        O = torch.empty_like(q)
    if LSE is None:
        LSE = torch.empty((S, H), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    # the library picks the scratch array of the current device: make it q's
    with torch.cuda.device(q.device):
        st = load().paged_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                              _ptr(seq_lens), int(block_size), _ptr(O), _ptr(LSE), S, H, d, nb, mb,
                                              float(scale), _dtype_code(q.dtype), _ptr(err_flag),
                                              _stream(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_attn_decode_noalloc (scratch limit %d bytes)" % ATTN_NOALLOC_SCRATCH_BYTES)
    return O, LSE


def paged_kv_append(k_new, v_new, seq_ids, positions, block_table, k_cache, v_cache, err_flag=None, stream=None):
    """Write new tokens' K/V ([T, H, d]) into the paged caches in place.
    seq_ids / positions: int32 [T]; block_table int32 [S, max_blocks_per_seq];
    caches [num_blocks, H, block_size, d].  See include/attn.h."""
    _check_cuda(k_new, v_new, seq_ids, positions, block_table, k_cache, v_cache, err_flag)
    T, H, d = k_new.shape
    if v_new.shape != k_new.shape or k_cache.shape != v_cache.shape or k_cache.shape[1] != H or \
            k_cache.shape[3] != d or k_new.dtype != k_cache.dtype or v_new.dtype != k_cache.dtype:
        raise ValueError("k_new/v_new [T, H, d] and caches [num_blocks, H, block_size, d] of one dtype")
    if seq_ids.dtype != torch.int32 or positions.dtype != torch.int32 or block_table.dtype != torch.int32:
        raise ValueError("seq_ids, positions and block_table must be int32")
    if tuple(seq_ids.shape) != (T,) or tuple(positions.shape) != (T,) or block_table.dim() != 2:
        raise ValueError("seq_ids and positions must be [T] and block_table [S, max_blocks_per_seq]")
    for t in (k_new, v_new, seq_ids, positions, block_table, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    _check_device(k_cache.device, k_new, v_new, seq_ids, positions, block_table, v_cache, err_flag)
    _check_err_flag(err_flag)
    with torch.cuda.device(k_cache.device):
        st = load().paged_kv_append(_ptr(k_new), _ptr(v_new), _ptr(seq_ids), _ptr(positions), T,
                                    _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(k_cache),
                                    _ptr(v_cache), k_cache.shape[0], H, d, k_cache.shape[2],
                                    _dtype_code(k_cache.dtype), _ptr(err_flag), _stream(stream, k_cache.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_kv_append")


def paged_block_copy(k_cache, v_cache, src_blocks, dst_blocks, err_flag=None, stream=None):
    """Copy physical blocks src -> dst in both caches (copy-on-write); the
    destinations must be distinct and not sources.  See include/attn.h."""
    _check_cuda(k_cache, v_cache, src_blocks, dst_blocks, err_flag)
    if src_blocks.dtype != torch.int32 or dst_blocks.dtype != torch.int32 or src_blocks.shape != dst_blocks.shape:
        raise ValueError("src_blocks and dst_blocks: int32 of one length")
    if k_cache.shape != v_cache.shape or not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("caches must be contiguous [num_blocks, H, block_size, d] of one shape")
    if v_cache.dtype != k_cache.dtype or k_cache.dim() != 4:
        raise ValueError("caches must be [num_blocks, H, block_size, d] of one dtype")
    _check_device(k_cache.device, v_cache, src_blocks, dst_blocks, err_flag)
    _check_err_flag(err_flag)
    nb, H, bs, d = k_cache.shape
    src, dst = src_blocks.contiguous(), dst_blocks.contiguous()
    with torch.cuda.device(k_cache.device):
        st = load().paged_block_copy(_ptr(k_cache), _ptr(v_cache), _ptr(src), _ptr(dst), src.numel(), nb, H, d,
                                     bs, _dtype_code(k_cache.dtype), _ptr(err_flag), _stream(stream, k_cache.device))
    if st != ATTN_OK:
        raise AttnError(st, "paged_block_copy")


def paged_cow_plan(block_table, ref_counts, free_list, free_count, write_seqs, write_blocks):
    """Copy-on-write planning on the host (include/attn.h): for the pending
    writes (write_seqs[i], write_blocks[i]), in order, every write into a
    block shared by several sequences takes a free block from the end of
    ``free_list[:free_count]``, the writer's entry of ``block_table`` is
    pointed at it and ``ref_counts`` are adjusted -- in place, on the
    caller's host arrays (numpy int32, or CPU int32 torch tensors, all
    contiguous).  Returns (src, dst, free_count): the copies to make with
    paged_block_copy before the writes, as int32 numpy arrays, and the new
    number of free blocks.  Raises AttnError (ATTN_ENOBLOCKS when the free
    list runs out, ATTN_EINVAL for an inconsistent table) with every array
    left as it was."""
    import numpy as np

    def host(x, name, ndim):
        if isinstance(x, torch.Tensor):
            if x.is_cuda:
                raise ValueError(f"{name} must be a host array (copy-on-write planning runs on the CPU)")
            x = x.numpy()
        if not isinstance(x, np.ndarray) or x.dtype != np.int32 or not x.flags.c_contiguous or x.ndim != ndim:
            raise ValueError(f"{name} must be a contiguous int32 host array with {ndim} dimension(s)")
        return x

    bt = host(block_table, "block_table", 2)
    rc = host(ref_counts, "ref_counts", 1)
    fl = host(free_list, "free_list", 1)
    ws = host(write_seqs, "write_seqs", 1)
    wb = host(write_blocks, "write_blocks", 1)
    if ws.shape != wb.shape:
        raise ValueError("write_seqs and write_blocks must have one length")
    if not 0 <= int(free_count) <= fl.shape[0]:
        raise ValueError("free_count must be within free_list")
    n = ws.shape[0]
    src = np.zeros(max(n, 1), dtype=np.int32)
    dst = np.zeros(max(n, 1), dtype=np.int32)
    fc = ctypes.c_int32(int(free_count))
    nc = ctypes.c_int32(0)
    addr = lambda a: a.ctypes.data if a.size else None  # noqa: E731
    st = load().paged_cow_plan(addr(bt), bt.shape[0], bt.shape[1], addr(rc), rc.shape[0], addr(fl),
                               ctypes.byref(fc), addr(ws), addr(wb), n, src.ctypes.data, dst.ctypes.data,
                               ctypes.byref(nc))
    if st != ATTN_OK:
        raise AttnError(st, "paged_cow_plan")
    return src[:nc.value].copy(), dst[:nc.value].copy(), int(fc.value)


def attn_selftest_wait_timeout(err_flag, result=None, stream=None) -> None:
    """Launch the bounded-wait self-test (attn.h): one CTA waits on an
    mbarrier phase nothing completes; after the 1 s limit the wait ORs
    ATTN_DEVERR_TIMEOUT into ``err_flag`` (int32 CUDA tensor) and writes 0 to
    ``result`` (int32 CUDA tensor, optional).  Asynchronous."""
    _check_cuda(err_flag, result)
    _check_err_flag(err_flag)
    _check_device(err_flag.device, result)
    if result is not None and (result.dtype != torch.int32 or result.numel() < 1):
        raise ValueError("result must be an int32 tensor with at least one element")
    with torch.cuda.device(err_flag.device):
        st = load().attn_selftest_wait_timeout(_ptr(err_flag), _ptr(result), _stream(stream, err_flag.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_wait_timeout")


def attn_selftest_exp2_poly(x, y=None, stream=None):
    """The prefill kernel's FMA-pipe 2^x on the fp32 CUDA tensor ``x``
    (attn.h: relative error <= 7.5e-5 on [-125, 8]).  Returns y (allocated
    when not given).  Asynchronous."""
    _check_cuda(x, y)
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 tensor")
    _check_device(x.device, y)
    _check_tensor(y, x.shape, torch.float32, "y")
    if y is None:
        y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        st = load().attn_selftest_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_exp2_poly")
    return y


def attn_read_error(err_flag, stream=None) -> int:
    """Synchronise the stream and return the device error bits (0 = none)."""
    _check_cuda(err_flag)
    _check_err_flag(err_flag)
    bits = ctypes.c_int32(0)
    with torch.cuda.device(err_flag.device):
        st = load().attn_read_error(_ptr(err_flag), ctypes.byref(bits), _stream(stream, err_flag.device))
    if st not in (ATTN_OK, ATTN_EDEVICE):
        raise AttnError(st, "attn_read_error")
    return int(bits.value)
