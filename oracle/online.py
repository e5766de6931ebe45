"""The pages' tiled algorithm, in plain numpy fp64 (small inputs only).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

This module walks the keys tile by tile the way the pages describe the method,
so that tests can check that the tiled method reaches the plain definition
(``oracle.attention``) for any tile size and any split of the key range:

* K-outer blocking: the keys of one (batch, kv-head) are visited in tiles of
  ``tile`` keys ("SmallQ FlashAttention for Ascend 910B", section "算法要点",
  K-outer blocking with a default block of 64 keys).
* Online softmax: two running quantities per query row, the current maximum
  m and the exponential sum l; when a tile raises the maximum, everything
  accumulated so far is rescaled by exp(m_old - m_new) ("昇腾CANN上的
  FlashAttention工程实战", section on tiling + online softmax; the CSDN
  "FlashAttention on Ascend CANN" post, section "在线 Softmax").
* Split-KV: the key range is cut into consecutive splits, each producing a
  normalised partial output and its log-sum-exp (the split-KV decode kernel
  of the MXFlashAttn PyPI page / sdist README); the partials are merged with
  log-sum-exp weights ("log-sum-exp trick", CSDN post).

Everything is fp64 and per row; nothing is fused or reordered beyond the
steps above.
"""
from __future__ import annotations

import math

import numpy as np


def _row_keys(n: int, Lq: int, i: int, causal: bool) -> int:
    """Number of leading keys visible to query i (bottom-right causal)."""
    last = n - 1
    if causal:
        last = min(last, i + n - Lq)
    return max(0, last + 1)


def split_partial(q_row, k_rows, v_rows, scale: float, lo: int, hi: int, visible: int,
                  tile: int):
    """Online softmax over keys [lo, hi) of one row, tile by tile.

    Returns (o_part, lse_part): the normalised partial output and the
    natural-log log-sum-exp of this split's visible scores; an empty split
    returns (zeros, -inf).
    """
    Dv = v_rows.shape[1]
    m = -math.inf
    l = 0.0
    acc = np.zeros(Dv, dtype=np.float64)
    hi = min(hi, visible)
    for t0 in range(lo, hi, tile):
        t1 = min(t0 + tile, hi)
        s = scale * (k_rows[t0:t1] @ q_row)          # scores of this tile
        m_new = max(m, float(np.max(s)))
        alpha = math.exp(m - m_new) if m != -math.inf else 0.0
        p = np.exp(s - m_new)
        l = alpha * l + float(np.sum(p))
        acc = alpha * acc + p @ v_rows[t0:t1]
        m = m_new
    if l == 0.0:
        return np.zeros(Dv, dtype=np.float64), -math.inf
    return acc / l, m + math.log(l)


def combine(o_parts, lse_parts):
    """Log-sum-exp weighted merge of split partials.

    L = ln sum_s exp(lse_s); O = sum_s exp(lse_s - L) O_s.  When every split is
    empty (all lse_s = -inf) the row is empty: O = 0, L = -inf.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    mx = float(np.max(lse_parts))
    Dv = np.asarray(o_parts[0]).shape[0]
    if mx == -math.inf:
        return np.zeros(Dv, dtype=np.float64), -math.inf
    w = np.exp(lse_parts - mx)
    L = mx + math.log(float(np.sum(w)))
    o = np.zeros(Dv, dtype=np.float64)
    for s in range(len(o_parts)):
        o += math.exp(lse_parts[s] - L) * np.asarray(o_parts[s], dtype=np.float64)
    return o, L


def attention_online(q, k, v, *, causal: bool = False, scale: float | None = None,
                     seqlens=None, tile: int = 64, split_bounds=None):
    """Tiled, split-KV attention over fp64 numpy arrays.

    q [B, Lq, Hq, Dqk], k [B, Lk, Hkv, Dqk], v [B, Lk, Hkv, Dv].
    split_bounds: optional callable (b, n) -> increasing list of split starts
    [0 = s_0 < s_1 < ... ] within [0, n); default is one split.
    Returns (o [B, Lq, Hq, Dv], lse [B, Hq, Lq]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Lq, Hq, Dqk = q.shape
    _, Lk, Hkv, _ = k.shape
    Dv = v.shape[3]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    o = np.zeros((B, Lq, Hq, Dv), dtype=np.float64)
    lse = np.full((B, Hq, Lq), -math.inf, dtype=np.float64)
    for b in range(B):
        n = int(seqlens[b]) if seqlens is not None else Lk
        starts = [0] if split_bounds is None else list(split_bounds(b, n))
        ends = starts[1:] + [n]
        for hq in range(Hq):
            hkv = hq // g
            for i in range(Lq):
                vis = _row_keys(n, Lq, i, causal)
                parts = [split_partial(q[b, i, hq], k[b, :, hkv], v[b, :, hkv], scale, lo, hi,
                                       vis, tile) for lo, hi in zip(starts, ends)]
                o[b, i, hq], lse[b, hq, i] = combine([p[0] for p in parts],
                                                     [p[1] for p in parts])
    return o, lse
