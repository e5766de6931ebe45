"""fp64 CPU oracle for decode / small-Q attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run anything in this package;
the product path (``decode_flashattention_b200``) never does, and this package
never imports it.  The two share no code: the oracle decodes fp16/bf16 bit
patterns itself and evaluates the plain definition

    O = softmax(Q K^T * scale) V,   scale = 1/sqrt(headDim) by default

("SmallQ FlashAttention for Ascend 910B", section "接口"; "昇腾CANN上的
FlashAttention工程实战", section on standard attention), with grouped-query
heads (hkv = hq // (Hq // Hkv)), a bottom-right aligned causal mask (key j is
visible to query i iff j <= i + n - Lq) and the natural-log log-sum-exp of the
scaled scores.  Rows with no visible key give O = 0, lse = -inf.

Modules:
  * ``attention_oracle.c`` -- the definition in C, fp64, threaded over rows.
  * ``online``             -- the pages' tiled online-softmax algorithm with
                              split-KV partials and a log-sum-exp combine, in
                              numpy fp64 (small inputs only).

Every function here is pinned by ``tests/test_oracle.py`` to closed forms,
invariants, a library routine (torch fp64 ``scaled_dot_product_attention``)
and exhaustive format checks; no function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

F16, BF16, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [
            p, p, p, p, p, p, ctypes.c_int,
            i64, i64, i64, i64, i64, i64, i64,
            p, ctypes.c_int, ctypes.c_double, i64, p, p, p, ctypes.c_int,
        ]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        _lib = lib
    return _lib


def f16_bits_to_f64(bits: int) -> float:
    return _load().oracle_f16_to_f64(bits)


def bf16_bits_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(bits)


def _as_raw(x):
    """Accept a numpy array (float16 / uint16-with-dtype / float64) or a CPU
    torch tensor (float16 / bfloat16 / float64); return (array, dtype code,
    element strides).  No value is converted: 16-bit inputs are passed as
    their bit patterns."""
    try:
        import torch  # torch is only used as a container here
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must live in host memory")
        code = {torch.float16: F16, torch.bfloat16: BF16, torch.float64: F64}.get(x.dtype)
        if code is None:
            raise TypeError(f"unsupported dtype {x.dtype}")
        strides = tuple(int(s) for s in x.stride())
        # the caller keeps the tensor alive; hand out its data pointer and strides
        return x, code, strides, x.data_ptr()
    a = np.asarray(x)
    if a.dtype == np.float16:
        code = F16
    elif a.dtype == np.float64:
        code = F64
    else:
        raise TypeError(f"unsupported numpy dtype {a.dtype} (bf16 must come as a torch tensor)")
    strides = tuple(s // a.itemsize for s in a.strides)
    return a, code, strides, a.ctypes.data


def attention(q, k, v, *, causal: bool = False, scale: float | None = None, seqlens=None,
              rows=None, nthreads: int | None = None):
    """Evaluate the definition.

    q: [B, Lq, Hq, Dqk]; k: [B, Lk, Hkv, Dqk]; v: [B, Lk, Hkv, Dv] (any strides,
    fp16 / bf16 / fp64, all the same type).  seqlens: optional int [B] with
    0 <= seqlens[b] <= Lk (the number of keys present for batch b).  rows:
    optional int array [n, 3] of (b, hq, i); when None every row is computed.

    Returns (o, lse): with rows=None, o is [B, Lq, Hq, Dv] and lse is
    [B, Hq, Lq]; with rows given, o is [n, Dv] and lse is [n].  Both fp64.
    """
    qa, qc, qs, qp = _as_raw(q)
    ka, kc, ks, kp = _as_raw(k)
    va, vc, vs, vp = _as_raw(v)
    if not (qc == kc == vc):
        raise TypeError("q, k, v must share one element type")
    if len(q.shape) != 4 or len(k.shape) != 4 or len(v.shape) != 4:
        raise ValueError("q, k, v must be 4-D [B, L, H, D]")
    B, Lq, Hq, Dqk = (int(s) for s in q.shape)
    Bk, Lk, Hkv, Dk = (int(s) for s in k.shape)
    Bv, Lv, Hv, Dv = (int(s) for s in v.shape)
    if (Bk, Dk) != (B, Dqk) or (Bv, Lv, Hv) != (Bk, Lk, Hkv) or Hq % Hkv:
        raise ValueError("inconsistent q/k/v shapes")
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    sl = None
    if seqlens is not None:
        sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(-1))
        if sl.shape[0] != B:
            raise ValueError("seqlens must have B entries")
    if rows is None:
        n = B * Hq * Lq
        rr = None
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rr.shape[0]
    o = np.empty((n, Dv), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    st = [np.asarray(s, dtype=np.int64) for s in (qs, ks, vs)]
    lib = _load()
    ret = lib.oracle_attention(
        qp, st[0].ctypes.data, kp, st[1].ctypes.data, vp, st[2].ctypes.data, qc,
        B, Lq, Hq, Lk, Hkv, Dqk, Dv,
        sl.ctypes.data if sl is not None else None, int(bool(causal)), float(scale),
        n, rr.ctypes.data if rr is not None else None, o.ctypes.data, lse.ctypes.data,
        int(max(1, nthreads)),
    )
    del qa, ka, va
    if ret == -1:
        raise ValueError("oracle_attention: invalid argument")
    if ret != 0:
        raise MemoryError("oracle_attention: out of memory or threads")
    if rows is None:
        o = o.reshape(B, Hq, Lq, Dv).transpose(0, 2, 1, 3).copy()
        lse = lse.reshape(B, Hq, Lq)
    return o, lse


def gather_pages(pages, block_table, seqlens):
    """Paged cache -> dense cache.

    pages: CPU torch tensor [num_blocks, page, H, D]; block_table: int array
    [B, max_blocks]; seqlens: int [B].  Returns a dense [B, max_blocks * page,
    H, D] tensor (same dtype, values copied unchanged) whose row j of batch b
    (j < seqlens[b]) is row j % page of block block_table[b, j // page] -- the
    block-table addressing of a paged K/V cache (FlashAttention's
    ``block_table`` convention, which the MXFlashAttn README's
    ``flash_attn_with_kvcache`` interface follows).  Rows at or past
    seqlens[b] are zero and never visible to the definition.
    """
    import torch  # a container and an index-copy primitive only

    bt = np.asarray(block_table, dtype=np.int64)
    sl = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    nb, page, H, D = (int(s) for s in pages.shape)
    B, mb = bt.shape
    out = torch.zeros((B, mb * page, H, D), dtype=pages.dtype)
    for b in range(B):
        n = int(min(max(sl[b], 0), mb * page))
        if n == 0:
            continue
        j = np.arange(n)
        blk = bt[b, j // page]
        if (blk < 0).any() or (blk >= nb).any():
            raise ValueError("block_table entry outside [0, num_blocks) within a sequence")
        out[b, :n] = pages[torch.from_numpy(blk), torch.from_numpy(j % page)]
    return out


def attention_paged(q, k_pages, v_pages, block_table, seqlens, *, causal: bool = False,
                    scale: float | None = None, rows=None, nthreads: int | None = None):
    """The definition over a paged K/V cache: gather_pages, then ``attention``
    with the cache lengths (keys past seqlens[b] are not present)."""
    k = gather_pages(k_pages, block_table, seqlens)
    v = gather_pages(v_pages, block_table, seqlens)
    sl = np.minimum(np.asarray(seqlens, dtype=np.int64).reshape(-1), k.shape[1]).clip(min=0)
    return attention(q, k, v, causal=causal, scale=scale, seqlens=sl, rows=rows, nthreads=nthreads)


def append_kv(k_cache, v_cache, k_new, v_new, seqlens, block_table=None):
    """KV append, written out: returns copies of the caches with token t of
    batch b written at position pos = seqlens[b] + t -- dense row pos of
    [B, Lmax, H, D], or (block_table given) row pos % page of block
    block_table[b, pos // page] of [num_blocks, page, H, D].  A position
    outside [0, capacity) or a block number outside [0, num_blocks) is not
    written.  CPU torch tensors in, values copied unchanged."""
    kc, vc = k_cache.clone(), v_cache.clone()
    sl = np.asarray(seqlens, dtype=np.int64).reshape(-1)
    B, Lnew = int(k_new.shape[0]), int(k_new.shape[1])
    if block_table is None:
        cap = int(kc.shape[1])
    else:
        bt = np.asarray(block_table, dtype=np.int64)
        page = int(kc.shape[1])
        cap = bt.shape[1] * page
    for b in range(B):
        for t in range(Lnew):
            pos = int(sl[b]) + t
            if pos < 0 or pos >= cap:
                continue
            if block_table is None:
                kc[b, pos] = k_new[b, t]
                vc[b, pos] = v_new[b, t]
            else:
                blk = int(bt[b, pos // page])
                if blk < 0 or blk >= kc.shape[0]:
                    continue
                kc[blk, pos % page] = k_new[b, t]
                vc[blk, pos % page] = v_new[b, t]
    return kc, vc


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, *, causal: bool = False, scale: float | None = None,
                     nthreads: int | None = None):
    """The definition within each packed sequence: q [total_q, Hq, Dqk],
    k [total_k, Hkv, Dqk], v [total_k, Hkv, Dv] (CPU); sequence b owns query
    tokens [cu_q[b], cu_q[b+1]) and key tokens [cu_k[b], cu_k[b+1]).  Returns
    (o [total_q, Hq, Dv], lse [Hq, total_q]), fp64."""
    cq = np.asarray(cu_seqlens_q, dtype=np.int64).reshape(-1)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64).reshape(-1)
    total_q, Hq = int(q.shape[0]), int(q.shape[1])
    Dv = int(v.shape[2])
    o = np.zeros((total_q, Hq, Dv), dtype=np.float64)
    lse = np.full((Hq, total_q), -np.inf, dtype=np.float64)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 <= q0:
            continue
        ob, lb = attention(q[q0:q1][None], k[k0:k1][None], v[k0:k1][None], causal=causal, scale=scale,
                           nthreads=nthreads)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse
