"""Shared helpers for the parity tests: oracle evaluation on host copies of the
device inputs, and the tolerance check.

Tolerances (written here, used by every parity test):
  * O: |gpu - oracle| <= max(TOL_O[dtype], 0.5 * ulp_dtype(|oracle|) + EPS_O * |oracle|),
    TOL_O = 2e-3 for fp16 and 1.6e-2 for bf16 outputs.  The second term
    only exceeds TOL_O where the output format cannot hold the oracle's value
    that closely: a correctly rounded fp16 / bf16 result is up to half an ulp
    away from the exact value (fp16: 1.95e-3 on [4, 8), 3.9e-3 on [8, 16);
    bf16: 1.56e-2 on [4, 8)), and EPS_O = 8 * 2^-24 is the margin of the
    kernels' fp32 accumulation ahead of that final rounding ("SmallQ
    FlashAttention for Ascend 910B", section "接口": fp32 accumulation).
  * lse: |gpu - oracle| / max(|oracle|, LSE_FLOOR) <= TOL_LSE = 1e-4.  The
    floor 1e-2 is where the fp32 score arithmetic's absolute error (about
    1e-6: a dot product of 16-bit values summed in fp32, then exp2 / log2 in
    fp32) reaches 1e-4 of the value; rows below it are checked against
    1e-6 absolute and counted.  Rows with no visible key must be exactly
    O = 0 and lse = -inf on both sides.

Every call of compare() records how many elements were judged by the
half-ulp term (and their largest error) and how many lse rows fell under
the floor; conftest.py prints the totals at the end of the session.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

TOL_O = {torch.float16: 2e-3, torch.bfloat16: 1.6e-2}
EPS_O = 8 * 2.0 ** -24
TOL_LSE = 1e-4
LSE_FLOOR = 1e-2

# running totals over the session (printed by conftest.py)
STATS = {"compares": 0, "o_elems": 0, "o_widened": 0, "o_widened_max_err": 0.0, "o_widened_max_excess": 0.0,
         "lse_rows": 0, "lse_floor_rows": 0, "lse_floor_max_abs": 0.0, "o_max_err": 0.0, "lse_max_rel": 0.0}
_MANT = {torch.float16: 10, torch.bfloat16: 7}
_MIN_EXP = {torch.float16: -14, torch.bfloat16: -126}


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    ax = np.maximum(np.abs(x), 1e-300)
    e = np.maximum(np.floor(np.log2(ax)), _MIN_EXP[dtype])
    return np.exp2(e - _MANT[dtype])


def o_bound(o_ref: np.ndarray, dtype) -> np.ndarray:
    """Per-element O bound: max(TOL_O, half an ulp of the output type at the
    oracle's value plus the fp32 accumulation margin)."""
    return np.maximum(TOL_O[dtype], 0.5 * ulp(o_ref, dtype) + EPS_O * np.abs(o_ref))


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    """Element-wise parity check; returns (max O error, max relative lse error)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    tol = o_bound(o_ref, dtype)
    err = np.abs(o_gpu - o_ref)
    bad = err > tol
    widened = tol > TOL_O[dtype]
    STATS["compares"] += 1
    STATS["o_elems"] += int(err.size)
    if err.size:
        STATS["o_max_err"] = max(STATS["o_max_err"], float(err.max()))
    if widened.any():
        STATS["o_widened"] += int(widened.sum())
        STATS["o_widened_max_err"] = max(STATS["o_widened_max_err"], float(err[widened].max()))
        STATS["o_widened_max_excess"] = max(STATS["o_widened_max_excess"],
                                            float((err[widened] - TOL_O[dtype]).max()))
    assert not bad.any(), (f"{what}: O mismatch at {np.argwhere(bad)[:5].tolist()} "
                           f"max err {err.max():.3e} (gpu {o_gpu[bad][:3]}, ref {o_ref[bad][:3]}, "
                           f"bound {tol[bad][:3]})")
    max_lse = 0.0
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        assert lse_gpu.shape == lse_ref.shape
        inf_ref = np.isinf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: empty-row pattern differs"
        fin = ~inf_ref
        if fin.any():
            d = np.abs(lse_gpu[fin] - lse_ref[fin])
            a = np.abs(lse_ref[fin])
            rel = d / np.maximum(a, LSE_FLOOR)
            max_lse = float(rel.max())
            low = a < LSE_FLOOR
            STATS["lse_rows"] += int(fin.sum())
            STATS["lse_max_rel"] = max(STATS["lse_max_rel"], float((d / np.maximum(a, 1e-300))[~low].max())
                                       if (~low).any() else 0.0)
            if low.any():
                STATS["lse_floor_rows"] += int(low.sum())
                STATS["lse_floor_max_abs"] = max(STATS["lse_floor_max_abs"], float(d[low].max()))
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
