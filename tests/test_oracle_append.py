"""Pins of the oracle's KV append (CPU only): appending then attending equals
the definition on the explicitly concatenated keys, for dense and paged
caches; positions past the capacity are not written."""
import numpy as np
import torch

import oracle


def test_append_then_attend_equals_concatenation():
    rng = np.random.default_rng(0)
    B, Lmax, Hq, Hkv, D, Lnew = 3, 20, 4, 2, 8, 3
    kc = torch.randn(B, Lmax, Hkv, D, dtype=torch.float64)
    vc = torch.randn(B, Lmax, Hkv, D, dtype=torch.float64)
    kn = torch.randn(B, Lnew, Hkv, D, dtype=torch.float64)
    vn = torch.randn(B, Lnew, Hkv, D, dtype=torch.float64)
    q = torch.randn(B, Lnew, Hq, D, dtype=torch.float64)
    sl = np.array([0, 5, 17])
    k2, v2 = oracle.append_kv(kc, vc, kn, vn, sl)
    for causal in (False, True):
        o, lse = oracle.attention(q, k2, v2, causal=causal, seqlens=sl + Lnew)
        for b in range(B):
            kcat = torch.cat([kc[b, :sl[b]], kn[b]])[None]
            vcat = torch.cat([vc[b, :sl[b]], vn[b]])[None]
            ob, lb = oracle.attention(q[b:b + 1], kcat, vcat, causal=causal)
            assert np.array_equal(o[b], ob[0]) and np.array_equal(lse[b], lb[0])
    # the cache keeps its other rows
    assert torch.equal(k2[1, :5], kc[1, :5]) and torch.equal(k2[1, 8:], kc[1, 8:])


def test_paged_append_writes_the_addressed_rows():
    nb, page, H, D = 6, 4, 1, 2
    kc = torch.zeros(nb, page, H, D, dtype=torch.float64)
    vc = torch.zeros(nb, page, H, D, dtype=torch.float64)
    kn = torch.arange(1, 1 + 2 * 3 * H * D, dtype=torch.float64).reshape(2, 3, H, D)
    vn = -kn
    table = np.array([[5, 2, -1], [0, 3, 1]])
    sl = [6, 11]  # batch 0: positions 6, 7, 8 -> block 2 rows 2, 3 and block -1 (skipped)
    k2, v2 = oracle.append_kv(kc, vc, kn, vn, sl, block_table=table)
    assert torch.equal(k2[2, 2], kn[0, 0]) and torch.equal(k2[2, 3], kn[0, 1])
    # batch 1: positions 11, 12, 13 -> block 1 row 3, then past the capacity 12
    assert torch.equal(k2[1, 3], kn[1, 0]) and torch.equal(v2[1, 3], vn[1, 0])
    written = (k2 != 0).any(-1).any(-1)
    assert int(written.sum()) == 3


def test_append_past_capacity_is_skipped():
    kc = torch.zeros(1, 4, 1, 2, dtype=torch.float64)
    k2, _ = oracle.append_kv(kc, kc, torch.ones(1, 3, 1, 2, dtype=torch.float64),
                             torch.ones(1, 3, 1, 2, dtype=torch.float64), [3])
    assert torch.equal(k2[0, 3], torch.ones(1, 2, dtype=torch.float64)) and int((k2 != 0).sum()) == 2
