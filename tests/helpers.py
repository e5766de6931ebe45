"""Shared helpers for the parity tests: oracle evaluation on host copies of the
device inputs, and the tolerance check.

Tolerances (written here, used by every parity test):
  * O: |gpu - oracle| <= max(TOL_O[dtype], ulp_dtype(|oracle|)), with TOL_O =
    2e-3 for fp16 and 1.6e-2 for bf16 outputs.  The second term only matters
    where the output format itself cannot hold the oracle's value that
    closely (|O| >= 4 in either format): there one unit in the last place of
    the output type is the representation limit of any implementation.
  * lse: |gpu - oracle| / max(|oracle|, 1) <= 1e-4; rows with no visible key
    must be exactly O = 0 and lse = -inf on both sides.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

TOL_O = {torch.float16: 2e-3, torch.bfloat16: 1.6e-2}
TOL_LSE = 1e-4
_MANT = {torch.float16: 10, torch.bfloat16: 7}
_MIN_EXP = {torch.float16: -14, torch.bfloat16: -126}


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    ax = np.maximum(np.abs(x), 1e-300)
    e = np.maximum(np.floor(np.log2(ax)), _MIN_EXP[dtype])
    return np.exp2(e - _MANT[dtype])


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    """Element-wise parity check; returns (max O error, max relative lse error)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    tol = np.maximum(TOL_O[dtype], ulp(o_ref, dtype))
    err = np.abs(o_gpu - o_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: O mismatch at {np.argwhere(bad)[:5].tolist()} "
                           f"max err {err.max():.3e} (gpu {o_gpu[bad][:3]}, ref {o_ref[bad][:3]})")
    max_lse = 0.0
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        assert lse_gpu.shape == lse_ref.shape
        inf_ref = np.isinf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: empty-row pattern differs"
        fin = ~inf_ref
        if fin.any():
            rel = np.abs(lse_gpu[fin] - lse_ref[fin]) / np.maximum(np.abs(lse_ref[fin]), 1.0)
            max_lse = float(rel.max())
            assert max_lse <= TOL_LSE, f"{what}: lse rel err {max_lse:.3e}"
    return float(err.max()) if err.size else 0.0, max_lse


def oracle_full(q, k, v, causal, scale=None, seqlens=None):
    """Oracle on host copies of whole device tensors (small cases)."""
    qc, kc, vc = (t.detach().cpu() for t in (q, k, v))
    sl = None if seqlens is None else seqlens.detach().cpu().numpy()
    return oracle.attention(qc, kc, vc, causal=causal, scale=scale, seqlens=sl)


def oracle_sampled(q, k, v, causal, rows, scale=None, seqlens=None):
    """Oracle for sampled output rows (b, hq, i) of a large device problem.

    Only the K/V slices of the sampled (batch, kv head) pairs are copied to the
    host: each pair becomes a sub-problem with one kv head and the g query
    heads of its group, so the grouped-query map is preserved."""
    B, Lq, Hq, _ = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    o_out = np.zeros((len(rows), v.shape[3]))
    lse_out = np.zeros(len(rows))
    groups = {}
    for idx, (b, hq, i) in enumerate(rows):
        groups.setdefault((int(b), int(hq) // g), []).append((idx, int(hq) % g, int(i)))
    for (b, hkv), items in groups.items():
        qs = q[b:b + 1, :, hkv * g:(hkv + 1) * g].detach().cpu()
        n = k.shape[1] if seqlens is None else int(seqlens[b])
        ks = k[b:b + 1, :max(n, 1), hkv:hkv + 1].detach().cpu()
        vs = v[b:b + 1, :max(n, 1), hkv:hkv + 1].detach().cpu()
        sl = None if seqlens is None else np.array([n], dtype=np.int32)
        rr = np.array([[0, h, i] for _, h, i in items], dtype=np.int64)
        o, lse = oracle.attention(qs, ks, vs, causal=causal, scale=scale, seqlens=sl, rows=rr)
        for j, (idx, _, _) in enumerate(items):
            o_out[idx] = o[j]
            lse_out[idx] = lse[j]
    return o_out, lse_out


def gather_rows(o, lse, rows):
    """Pick sampled rows (b, hq, i) out of device results."""
    oc = o.detach().float().cpu().numpy()
    lc = lse.detach().cpu().numpy() if lse is not None else None
    og = np.stack([oc[b, i, h] for b, h, i in rows])
    lg = None if lc is None else np.array([lc[b, h, i] for b, h, i in rows])
    return og, lg


def sample_rows(B, Hq, Lq, n, seed):
    rng = np.random.default_rng(seed)
    rows = {(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(Lq))) for _ in range(n)}
    # always include the corners
    rows |= {(0, 0, 0), (B - 1, Hq - 1, Lq - 1), (0, Hq - 1, Lq - 1)}
    return sorted(rows)


def o_to_numpy(o):
    return o.detach().float().cpu().numpy()


def lse_to_numpy(lse):
    return lse.detach().cpu().numpy()
