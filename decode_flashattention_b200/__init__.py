"""decode_flashattention_b200 -- decode / small-Q FlashAttention for B200 (sm_100a).

A thin ctypes binding over ``libfa_b200.so`` (C ABI: ``include/fa.h``).  The
binding only marshals arguments: it builds tensor descriptors, allocates the
output / LSE / workspace tensors with PyTorch when the caller does not pass
them, and hands the current CUDA stream to the library.  Every step of the
attention itself runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing or unloadable library raises at first use.

Public calls (names follow the FlashAttention API the pages describe:
``flash_attn_func`` / ``flash_attn_with_kvcache`` in the MXFlashAttn README):

* ``fa_fwd(q, k, v, causal, scale)`` / ``flash_attn_func`` -- q [B, Lq, Hq, D],
  k/v [B, Lk, Hkv, D]; returns (o, lse).
* ``fa_decode_kvcache(q, k_cache, v_cache, cache_seqlens, ...)`` /
  ``flash_attn_with_kvcache`` -- attention against the first
  ``cache_seqlens[b]`` keys of each batch's cache.
* ``hld_as_blhd(x)`` -- view a [H, L, D] tensor as [1, L, H, D] (no copy).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "FaError", "fa_fwd", "fa_decode_kvcache", "fa_decode_kvcache_paged", "paged_workspace_size",
    "fa_decode_kvcache_append", "fa_fwd_varlen", "flash_attn_varlen_func",
    "flash_attn_func", "flash_attn_with_kvcache",
    "fwd_workspace_size", "kvcache_workspace_size", "hld_as_blhd", "check_status",
    "last_dispatch", "force_variant", "force_tcgen05_form", "test_stall_next_call", "profile_enable", "profile_read", "launch_count",
    "library_path", "load_library", "schedule", "VARIANT_AUTO", "VARIANT_MMA", "VARIANT_SCALAR", "VARIANT_TCGEN05",
    "VARIANT_TCGEN05_SPLIT",
    "TCGEN05_AUTO", "TCGEN05_TWO_TILES", "TCGEN05_ONE_TILE_MMA",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfa_b200.so")
_lib = None

VARIANT_AUTO, VARIANT_MMA, VARIANT_SCALAR, VARIANT_TCGEN05, VARIANT_TCGEN05_SPLIT = 0, 1, 2, 3, 4
TCGEN05_AUTO, TCGEN05_TWO_TILES, TCGEN05_ONE_TILE_MMA = 0, 2, 3  # form 1 is retired
_STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_WORKSPACE",
           4: "FA_ERR_CUDA", 5: "FA_ERR_TIMEOUT"}
_DTYPE = {torch.float16: 0, torch.bfloat16: 1}


class FaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class FaDispatchInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "variant", "grid", "block", "smem_bytes", "tile_keys", "stages", "rows_per_cta", "units",
        "min_share_tiles", "combine_launched")] + [("work_tiles", ctypes.c_int64), ("tcgen05_form", ctypes.c_int32),
                                                   ("reserved", ctypes.c_int32)]


class FaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libfa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m decode_flashattention_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.POINTER
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    T = P(FaTensor)
    sig = {
        "fa_fwd": (i32, [T, T, T, T, vp, i32, f32, i32, vp, sz, vp]),
        "fa_fwd_workspace_size": (i32, [T, T, T, i32, i32, P(sz)]),
        "fa_decode_kvcache": (i32, [T, T, T, vp, T, vp, i32, i32, f32, vp, sz, vp]),
        "fa_decode_kvcache_workspace_size": (i32, [T, T, T, i32, P(sz)]),
        "fa_decode_kvcache_paged": (i32, [T, T, T, vp, ctypes.c_int64, i32, vp, T, vp, i32, i32, f32, vp, sz, vp]),
        "fa_decode_kvcache_paged_workspace_size": (i32, [T, T, T, i32, i32, P(sz)]),
        "fa_fwd_varlen": (i32, [T, T, T, vp, vp, i32, i32, i32, T, vp, i32, f32, i32, vp, sz, vp]),
        "fa_fwd_varlen_workspace_size": (i32, [T, T, T, i32, i32, i32, i32, P(sz)]),
        "fa_decode_kvcache_append": (i32, [T, T, T, T, T, vp, ctypes.c_int64, i32, vp, T, vp, i32, i32, f32, vp,
                                           sz, vp]),
        "fa_check_status": (i32, [vp]),
        "fa_last_error": (ctypes.c_char_p, []),
        "fa_last_dispatch": (None, [P(FaDispatchInfo)]),
        "fa_force_variant": (i32, [i32]),
        "fa_force_tcgen05_form": (i32, [i32]),
        "fa_test_stall_next_call": (i32, [ctypes.c_ulonglong]),
        "fa_profile_enable": (i32, [i32]),
        "fa_profile_read": (i32, [P(ctypes.c_double), P(ctypes.c_int64), P(ctypes.c_double),
                                  P(ctypes.c_int64)]),
        "fa_schedule": (i32, [i32, i32, i32, i32, i32, i32, vp, i32, i32, i32, i32, i32, P(ctypes.c_int64),
                              P(ctypes.c_int64), vp, vp, vp, ctypes.c_int64]),
        "fa_launch_count": (ctypes.c_int64, []),
        "fa_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        msg = load_library().fa_last_error().decode(errors="replace")
        raise FaError(status, msg)


def _desc(t: torch.Tensor, name: str) -> FaTensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != 4:
        raise ValueError(f"{name} must be 4-D [B, L, H, D], got {tuple(t.shape)}")
    if t.dtype not in _DTYPE:
        raise TypeError(f"{name}: dtype {t.dtype} is not float16/bfloat16")
    d = FaTensor()
    d.data = t.data_ptr() if t.numel() else None
    d.dtype = _DTYPE[t.dtype]
    for i in range(4):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def hld_as_blhd(x: torch.Tensor) -> torch.Tensor:
    """View a [H, L, D] tensor as [1, L, H, D] (strides {H*L*D, D, L*D, 1})."""
    if x.dim() != 3:
        raise ValueError("expected [H, L, D]")
    return x.unsqueeze(0).permute(0, 2, 1, 3)


def _stream_ptr(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _cuda_inputs(*ts):
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise ValueError("inputs must be CUDA tensors")
        if t.device != dev:
            raise ValueError("inputs must live on one device")
    return dev


def fwd_workspace_size(q, k, v, causal=False, num_splits=0) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    with torch.cuda.device(q.device):
        _check(lib.fa_fwd_workspace_size(_desc(q, "q"), _desc(k, "k"), _desc(v, "v"), int(bool(causal)),
                                         int(num_splits), ctypes.byref(n)))
    return n.value


def kvcache_workspace_size(q, k_cache, v_cache, num_splits=0) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    with torch.cuda.device(q.device):
        _check(lib.fa_decode_kvcache_workspace_size(_desc(q, "q"), _desc(k_cache, "k_cache"),
                                                    _desc(v_cache, "v_cache"), int(num_splits),
                                                    ctypes.byref(n)))
    return n.value


def _outputs(q, Dv, out, lse, want_lse):
    B, Lq, Hq, _ = q.shape
    if out is None:
        out = torch.empty((B, Lq, Hq, Dv), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or tuple(lse.shape) != (B, Hq, Lq)):
        raise ValueError("lse must be a contiguous float32 [B, Hq, Lq] tensor")
    return out, lse


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")
    return workspace, workspace.numel() * workspace.element_size()


def fa_fwd(q, k, v, causal=False, scale=None, num_splits=0, out=None, lse=None, workspace=None,
           return_lse=True):
    """O = softmax(Q K^T * scale) V over dense q [B, Lq, Hq, Dqk], k [B, Lk, Hkv, Dqk],
    v [B, Lk, Hkv, Dv]; causal masks bottom-right aligned.  Returns (o, lse)."""
    lib = load_library()
    dev = _cuda_inputs(q, k, v)
    out, lse = _outputs(q, v.shape[3], out, lse, return_lse)
    with torch.cuda.device(dev):
        nbytes = fwd_workspace_size(q, k, v, causal, num_splits)
        ws, ws_bytes = _workspace(nbytes, dev, workspace)
        _check(lib.fa_fwd(_desc(q, "q"), _desc(k, "k"), _desc(v, "v"), _desc(out, "o"),
                          ctypes.c_void_p(lse.data_ptr() if lse is not None else None),
                          int(bool(causal)), float(scale or 0.0), int(num_splits),
                          ctypes.c_void_p(ws.data_ptr() if ws is not None else None), ws_bytes,
                          _stream_ptr(q)))
    return out, lse


def fa_decode_kvcache(q, k_cache, v_cache, cache_seqlens, causal=False, scale=None, num_splits=0,
                      out=None, lse=None, workspace=None, return_lse=True):
    """Attention of q [B, Lq, Hq, Dqk] against the first cache_seqlens[b] keys of
    k_cache / v_cache [B, Lmax, Hkv, D] (cache_seqlens: CUDA int32 [B])."""
    lib = load_library()
    dev = _cuda_inputs(q, k_cache, v_cache, cache_seqlens)
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.dim() != 1 or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 [B] tensor")
    if cache_seqlens.shape[0] != q.shape[0]:
        raise ValueError("cache_seqlens must have B entries")
    out, lse = _outputs(q, v_cache.shape[3], out, lse, return_lse)
    with torch.cuda.device(dev):
        nbytes = kvcache_workspace_size(q, k_cache, v_cache, num_splits)
        ws, ws_bytes = _workspace(nbytes, dev, workspace)
        _check(lib.fa_decode_kvcache(_desc(q, "q"), _desc(k_cache, "k_cache"), _desc(v_cache, "v_cache"),
                                     ctypes.c_void_p(cache_seqlens.data_ptr()), _desc(out, "o"),
                                     ctypes.c_void_p(lse.data_ptr() if lse is not None else None),
                                     int(num_splits), int(bool(causal)), float(scale or 0.0),
                                     ctypes.c_void_p(ws.data_ptr() if ws is not None else None),
                                     ws_bytes, _stream_ptr(q)))
    return out, lse


def paged_workspace_size(q, k_pages, v_pages, max_blocks_per_seq, num_splits=0) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    with torch.cuda.device(q.device):
        _check(lib.fa_decode_kvcache_paged_workspace_size(_desc(q, "q"), _desc(k_pages, "k_pages"),
                                                          _desc(v_pages, "v_pages"), int(max_blocks_per_seq),
                                                          int(num_splits), ctypes.byref(n)))
    return n.value


def fa_decode_kvcache_paged(q, k_pages, v_pages, block_table, cache_seqlens, causal=False, scale=None,
                            num_splits=0, out=None, lse=None, workspace=None, return_lse=True):
    """Attention of q [B, Lq, Hq, Dqk] against a paged cache: k_pages / v_pages
    [num_blocks, page, Hkv, D], block_table CUDA int32 [B, max_blocks_per_seq]
    (row stride free, unit column stride), cache_seqlens CUDA int32 [B]; key j
    of batch b is row j % page of block block_table[b, j // page]."""
    lib = load_library()
    dev = _cuda_inputs(q, k_pages, v_pages, block_table, cache_seqlens)
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.dim() != 1 or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 [B] tensor")
    if cache_seqlens.shape[0] != q.shape[0]:
        raise ValueError("cache_seqlens must have B entries")
    if (block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != q.shape[0]
            or block_table.stride(1) != 1):
        raise ValueError("block_table must be an int32 [B, max_blocks_per_seq] tensor with unit column stride")
    out, lse = _outputs(q, v_pages.shape[3], out, lse, return_lse)
    mb = block_table.shape[1]
    with torch.cuda.device(dev):
        nbytes = paged_workspace_size(q, k_pages, v_pages, mb, num_splits)
        ws, ws_bytes = _workspace(nbytes, dev, workspace)
        _check(lib.fa_decode_kvcache_paged(
            _desc(q, "q"), _desc(k_pages, "k_pages"), _desc(v_pages, "v_pages"),
            ctypes.c_void_p(block_table.data_ptr()), int(block_table.stride(0)), int(mb),
            ctypes.c_void_p(cache_seqlens.data_ptr()), _desc(out, "o"),
            ctypes.c_void_p(lse.data_ptr() if lse is not None else None), int(num_splits), int(bool(causal)),
            float(scale or 0.0), ctypes.c_void_p(ws.data_ptr() if ws is not None else None), ws_bytes,
            _stream_ptr(q)))
    return out, lse


def fa_decode_kvcache_append(q, k_new, v_new, k_cache, v_cache, cache_seqlens, block_table=None, causal=False,
                             scale=None, num_splits=0, out=None, lse=None, workspace=None, return_lse=True):
    """Write k_new / v_new [B, Lnew, Hkv, D] into the cache at positions
    cache_seqlens[b] + t (dense k_cache [B, Lmax, Hkv, D], or paged
    [num_blocks, page, Hkv, D] with block_table), then attend over
    cache_seqlens[b] + Lnew keys.  cache_seqlens is not modified."""
    lib = load_library()
    dev = _cuda_inputs(q, k_new, v_new, k_cache, v_cache, cache_seqlens)
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.dim() != 1 or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 [B] tensor")
    if cache_seqlens.shape[0] != q.shape[0]:
        raise ValueError("cache_seqlens must have B entries")
    if block_table is not None:
        if (block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != q.shape[0]
                or block_table.stride(1) != 1 or block_table.device != dev):
            raise ValueError("block_table must be a CUDA int32 [B, max_blocks_per_seq] tensor, unit column stride")
        mb, bts, btp = block_table.shape[1], block_table.stride(0), block_table.data_ptr()
    else:
        mb, bts, btp = 0, 0, None
    out, lse = _outputs(q, v_cache.shape[3], out, lse, return_lse)
    with torch.cuda.device(dev):
        if block_table is not None:
            nbytes = paged_workspace_size(q, k_cache, v_cache, mb, num_splits)
        else:
            nbytes = kvcache_workspace_size(q, k_cache, v_cache, num_splits)
        ws, ws_bytes = _workspace(nbytes, dev, workspace)
        _check(lib.fa_decode_kvcache_append(
            _desc(q, "q"), _desc(k_new, "k_new"), _desc(v_new, "v_new"), _desc(k_cache, "k_cache"),
            _desc(v_cache, "v_cache"), ctypes.c_void_p(btp), int(bts), int(mb),
            ctypes.c_void_p(cache_seqlens.data_ptr()), _desc(out, "o"),
            ctypes.c_void_p(lse.data_ptr() if lse is not None else None), int(num_splits), int(bool(causal)),
            float(scale or 0.0), ctypes.c_void_p(ws.data_ptr() if ws is not None else None), ws_bytes,
            _stream_ptr(q)))
    return out, lse


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False, scale=None,
                  num_splits=0, out=None, lse=None, workspace=None, return_lse=True):
    """Attention within packed variable-length sequences: q [total_q, Hq, Dqk],
    k [total_k, Hkv, Dqk], v [total_k, Hkv, Dv] (3-D, or 4-D with a leading 1),
    cu_seqlens_q / cu_seqlens_k CUDA int32 [batch + 1].  Returns
    (o [total_q, Hq, Dv] in q's rank, lse [Hq, total_q])."""
    lib = load_library()
    dev = _cuda_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k)
    for name, cu in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if cu.dtype != torch.int32 or cu.dim() != 1 or not cu.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 [batch + 1] tensor")
    if cu_seqlens_k.shape[0] != cu_seqlens_q.shape[0]:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    batch = cu_seqlens_q.shape[0] - 1
    squeeze = q.dim() == 3
    q4, k4, v4 = (t.unsqueeze(0) if t.dim() == 3 else t for t in (q, k, v))
    total_q, Hq = q4.shape[1], q4.shape[2]
    if out is None:
        out = torch.empty((1, total_q, Hq, v4.shape[3]), dtype=q.dtype, device=dev)
    o4 = out.unsqueeze(0) if out.dim() == 3 else out
    if lse is None and return_lse:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=dev)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or tuple(lse.shape) != (Hq, total_q)):
        raise ValueError("lse must be a contiguous float32 [Hq, total_q] tensor")
    with torch.cuda.device(dev):
        n = ctypes.c_size_t(0)
        _check(lib.fa_fwd_varlen_workspace_size(_desc(q4, "q"), _desc(k4, "k"), _desc(v4, "v"), int(batch),
                                                int(max_seqlen_q), int(max_seqlen_k), int(num_splits),
                                                ctypes.byref(n)))
        ws, ws_bytes = _workspace(n.value, dev, workspace)
        _check(lib.fa_fwd_varlen(
            _desc(q4, "q"), _desc(k4, "k"), _desc(v4, "v"), ctypes.c_void_p(cu_seqlens_q.data_ptr()),
            ctypes.c_void_p(cu_seqlens_k.data_ptr()), int(batch), int(max_seqlen_q), int(max_seqlen_k),
            _desc(o4, "o"), ctypes.c_void_p(lse.data_ptr() if lse is not None else None), int(bool(causal)),
            float(scale or 0.0), int(num_splits), ctypes.c_void_p(ws.data_ptr() if ws is not None else None),
            ws_bytes, _stream_ptr(q)))
    return (o4[0] if squeeze and out.dim() == 4 else out), lse


def flash_attn_varlen_func(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                           softmax_scale=None, return_attn_probs=False):
    o, lse = fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=causal,
                           scale=softmax_scale, return_lse=return_attn_probs)
    return (o, lse) if return_attn_probs else o


def flash_attn_func(q, k, v, causal=False, softmax_scale=None, return_lse=False):
    o, lse = fa_fwd(q, k, v, causal=causal, scale=softmax_scale, return_lse=return_lse)
    return (o, lse) if return_lse else o


def flash_attn_with_kvcache(q, k_cache, v_cache, cache_seqlens, causal=False, softmax_scale=None,
                            num_splits=0, return_softmax_lse=False, block_table=None, k=None, v=None):
    """Dense cache ([B, Lmax, Hkv, D]) or, with block_table, a paged one
    ([num_blocks, page, Hkv, D]); with k / v ([B, Lnew, Hkv, D]) those tokens
    are appended to the cache first."""
    if k is not None or v is not None:
        if k is None or v is None:
            raise ValueError("k and v are appended together")
        o, lse = fa_decode_kvcache_append(q, k, v, k_cache, v_cache, cache_seqlens, block_table=block_table,
                                          causal=causal, scale=softmax_scale, num_splits=num_splits,
                                          return_lse=return_softmax_lse)
    elif block_table is None:
        o, lse = fa_decode_kvcache(q, k_cache, v_cache, cache_seqlens, causal=causal, scale=softmax_scale,
                                   num_splits=num_splits, return_lse=return_softmax_lse)
    else:
        o, lse = fa_decode_kvcache_paged(q, k_cache, v_cache, block_table, cache_seqlens, causal=causal,
                                         scale=softmax_scale, num_splits=num_splits,
                                         return_lse=return_softmax_lse)
    return (o, lse) if return_softmax_lse else o


def check_status(device=None):
    """Synchronise the current stream and raise FaError if a kernel timed out."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib.fa_check_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))


def last_dispatch() -> dict:
    info = FaDispatchInfo()
    load_library().fa_last_dispatch(ctypes.byref(info))
    return {n: getattr(info, n) for n, _ in FaDispatchInfo._fields_ if n != "reserved"}


def force_variant(variant: int):
    _check(load_library().fa_force_variant(int(variant)))


def test_stall_next_call(wait_limit_ns: int):
    """Test hook: the next split-KV call leaves one pipeline stage empty and
    bounds its waits by wait_limit_ns, so it ends with FA_ERR_TIMEOUT in the
    device status word (read by check_status)."""
    _check(load_library().fa_test_stall_next_call(int(wait_limit_ns)))


def force_tcgen05_form(form: int):
    """Force the tcgen05 kernel's form (TCGEN05_AUTO restores the library's choice)."""
    _check(load_library().fa_force_tcgen05_form(int(form)))


def profile_enable(on: bool):
    _check(load_library().fa_profile_enable(int(bool(on))))


def profile_read() -> dict:
    mm, cm = ctypes.c_double(), ctypes.c_double()
    mn, cn = ctypes.c_int64(), ctypes.c_int64()
    _check(load_library().fa_profile_read(ctypes.byref(mm), ctypes.byref(mn), ctypes.byref(cm),
                                          ctypes.byref(cn)))
    return {"main_ms": mm.value, "main_launches": mn.value, "combine_ms": cm.value,
            "combine_launches": cn.value}


def schedule(B, Lq, Hq, Hkv, Lk, causal, seqlens=None, num_ctas=148, min_share=2, tile_keys=128,
             rows_per_cta=8, seg_cost=0):
    """Host copy of the kernels' work partition (see fa_schedule in include/fa.h).
    Returns dict(work_tiles, ctas_used, unit_tiles, unit_first_cta, unit_last_cta)."""
    import numpy as np

    g = Hq // Hkv
    units = B * ((g * Lq + rows_per_cta - 1) // rows_per_cta) * Hkv
    tiles = np.zeros(units, dtype=np.int32)
    first = np.zeros(units, dtype=np.int64)
    last = np.zeros(units, dtype=np.int64)
    sl = None if seqlens is None else np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    W, P = ctypes.c_int64(), ctypes.c_int64()
    _check(load_library().fa_schedule(
        int(B), int(Lq), int(Hq), int(Hkv), int(Lk), int(bool(causal)),
        ctypes.c_void_p(sl.ctypes.data if sl is not None else None), int(num_ctas), int(min_share),
        int(tile_keys), int(rows_per_cta), int(seg_cost), ctypes.byref(W), ctypes.byref(P),
        ctypes.c_void_p(tiles.ctypes.data),
        ctypes.c_void_p(first.ctypes.data), ctypes.c_void_p(last.ctypes.data), units))
    return {"work_tiles": W.value, "ctas_used": P.value, "unit_tiles": tiles,
            "unit_first_cta": first, "unit_last_cta": last}


def launch_count() -> int:
    return int(load_library().fa_launch_count())


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
