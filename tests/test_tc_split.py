"""GPU parity of the tcgen05 split-KV kernel (FA_VARIANT_TCGEN05_SPLIT) against
the fp64 oracle, through the C ABI.

The kernel takes the g * Lq packed rows of a GQA group (with their
speculative query positions) as one unit of 16, 32 or 64 rows, so it runs
whenever g * Lq > 8.  Covered: row counts on both sides of every block size
(9 .. 128 rows, the last blocks ragged), head dims 64 .. 192 / 128, fp16 and
bf16, causal and not, key lengths at tile edges, the KV-cache call with
NaN-poisoned tails and empty caches, paged caches, packed variable-length
inputs, KV append, split counts, agreement with the mma.sync kernel's 8-row
blocks, the dispatch record, and the batched GQA-8 speculative decode at
full size on sampled rows.
"""
import dataclasses

import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import (compare, gather_rows, lse_to_numpy, o_to_numpy, oracle_full, oracle_sampled,
                     sample_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _tc_variant():
    # the shapes here are small, where the library itself would choose the
    # mma.sync kernel: force the tcgen05 split-KV kernel
    fa.force_variant(fa.VARIANT_TCGEN05_SPLIT)
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


def _expect_rows(R):
    return 16 if R <= 16 else (32 if R <= 32 else 64)


def _fwd(w, num_splits=0):
    q, k, v, sl = wl.make_inputs(w, DEV)
    if w.call == "kvcache":
        o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=w.causal, num_splits=num_splits)
    else:
        o, lse = fa.fa_fwd(q, k, v, causal=w.causal, num_splits=num_splits)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    ro, rl = oracle_full(q, k, v, w.causal, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, w.name)
    return d, (q, k, v, sl), (o, lse)


# (g, Lq): packed rows 9 .. 128 -- below, at and past each block size
ROWS = [(3, 3), (2, 8), (8, 2), (16, 1), (17, 1), (4, 5), (8, 4), (32, 1), (11, 3), (8, 6), (16, 4), (8, 8),
        (13, 5), (16, 8)]


@pytest.mark.parametrize("g,lq", ROWS, ids=[f"g{g}q{lq}" for g, lq in ROWS])
@pytest.mark.parametrize("causal", [False, True])
def test_row_counts(g, lq, causal):
    w = wl.Workload("tcs_rows", "fwd", "blhd", torch.bfloat16, B=2, Lq=lq, Hq=2 * g, Hkv=2, Lk=700, Dqk=128,
                    Dv=128, causal=causal, seed=100 * g + lq)
    d, _, _ = _fwd(w)
    assert d["variant"] == fa.VARIANT_TCGEN05_SPLIT
    assert d["rows_per_cta"] == _expect_rows(g * lq)


SWEEP = []
_rng = np.random.default_rng(515)
for kv in (1, 2, 100, 127, 128, 129, 1000, 2500):
    for dims in ((64, 64), (128, 128), (192, 128), (96, 40), (160, 128)):
        g, lq = ROWS[int(_rng.integers(len(ROWS) - 1))]
        dt = torch.float16 if _rng.random() < 0.5 else torch.bfloat16
        SWEEP.append((kv, g, lq, dims, dt, bool(_rng.random() < 0.5)))


@pytest.mark.parametrize("kv,g,lq,dims,dt,causal", SWEEP,
                         ids=[f"kv{a}-g{b}q{c}-d{d[0]}_{d[1]}-{str(e)[6:]}-c{int(f)}" for a, b, c, d, e, f in SWEEP])
def test_shape_sweep(kv, g, lq, dims, dt, causal):
    w = wl.Workload("tcs_sweep", "fwd", "blhd", dt, B=2, Lq=lq, Hq=g, Hkv=1, Lk=kv, Dqk=dims[0], Dv=dims[1],
                    causal=causal, seed=kv + 13 * g + lq)
    d, _, _ = _fwd(w)
    assert d["variant"] == fa.VARIANT_TCGEN05_SPLIT


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_kvcache_poisoned_tails_and_edges(causal, dt):
    w = wl.Workload("tcs_kv", "kvcache", "blhd", dt, B=8, Lq=4, Hq=16, Hkv=2, Lk=600, Dqk=128, Dv=128,
                    causal=causal, seed=31 + causal)
    q, k, v, _ = wl.make_inputs(dataclasses.replace(w, call="fwd"), DEV)
    sl = torch.tensor([0, 1, 3, 127, 128, 129, 513, 600], dtype=torch.int32)
    for b in range(w.B):
        k[b, int(sl[b]):] = float("nan")
        v[b, int(sl[b]):] = float("nan")
    o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=causal)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05_SPLIT
    ro, rl = oracle_full(q, k, v, causal, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, "tcs kvcache")


@pytest.mark.parametrize("num_splits", [1, 2, 5, 64])
def test_split_counts(num_splits):
    w = wl.Workload("tcs_splits", "kvcache", "blhd", torch.bfloat16, B=3, Lq=4, Hq=32, Hkv=4, Lk=3000, Dqk=128,
                    Dv=128, causal=True, seed=71, seqlen_lo=1, seqlen_hi=3000)
    _fwd(w, num_splits=num_splits)


def test_agrees_with_mma_blocks_of_8():
    """The same call on the mma.sync kernel (row blocks of 8, K / V read once
    per block) and on the tcgen05 kernel (one block): both within the bound of
    the oracle, and of each other."""
    w = wl.Workload("tcs_vs_mma", "fwd", "blhd", torch.float16, B=2, Lq=8, Hq=16, Hkv=2, Lk=1500, Dqk=128, Dv=128,
                    causal=True, seed=5)
    _, (q, k, v, _), (o1, l1) = _fwd(w)
    fa.force_variant(fa.VARIANT_MMA)
    o2, l2 = fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["rows_per_cta"] == 8
    compare(o_to_numpy(o2), lse_to_numpy(l2), o_to_numpy(o1).astype(np.float64), lse_to_numpy(l1), w.dtype,
            "mma vs tcgen05 split")


@pytest.mark.parametrize("page", [16, 64, 256])
def test_paged(page):
    w = wl.Workload("tcs_paged", "paged", "blhd", torch.bfloat16, B=5, Lq=4, Hq=16, Hkv=2, Lk=900, Dqk=128,
                    Dv=128, causal=True, seed=page, seqlen_lo=0, seqlen_hi=900, page=page)
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV, poison=True)
    o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05_SPLIT
    ro, rl = oracle.attention_paged(q.cpu(), kp.cpu(), vp.cpu(), bt.cpu().numpy(), sl.numpy(), causal=True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, f"tcs paged{page}")


def test_varlen():
    lq, lk = [1, 8, 3, 5, 0, 8], [700, 64, 1, 300, 50, 129]
    Hq, Hkv, dt = 16, 2, torch.float16
    g = torch.Generator(device=DEV).manual_seed(9)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    q = torch.randn(int(cq[-1]), Hq, 128, generator=g, device=DEV).to(dt)
    k = torch.randn(int(ck[-1]), Hkv, 128, generator=g, device=DEV).to(dt)
    v = torch.randn(int(ck[-1]), Hkv, 128, generator=g, device=DEV).to(dt)
    o, lse = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), max(lq), max(lk), causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05_SPLIT
    ro, rl = oracle.attention_varlen(q.cpu(), k.cpu(), v.cpu(), cq.numpy(), ck.numpy(), causal=True)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, dt, "tcs varlen")


def test_append():
    w = wl.Workload("tcs_app", "kvcache", "blhd", torch.bfloat16, B=4, Lq=4, Hq=16, Hkv=2, Lk=700, Dqk=128,
                    Dv=128, causal=True, seed=44, seqlen_lo=0, seqlen_hi=696)
    q, kc, vc, sl = wl.make_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(45)
    kn = torch.randn(4, 4, 2, 128, generator=g, device=DEV).to(w.dtype)
    vn = torch.randn(4, 4, 2, 128, generator=g, device=DEV).to(w.dtype)
    k0, v0 = kc.clone(), vc.clone()
    o, lse = fa.fa_decode_kvcache_append(q, kn, vn, kc, vc, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05_SPLIT
    kr, vr = oracle.append_kv(k0.cpu(), v0.cpu(), kn.cpu(), vn.cpu(), sl.numpy())
    assert torch.equal(kc.cpu(), kr) and torch.equal(vc.cpu(), vr)
    ro, rl = oracle.attention(q.cpu(), kr, vr, causal=True, seqlens=np.minimum(sl.numpy() + 4, 700))
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "tcs append")


def test_determinism_bitwise():
    w = wl.Workload("tcs_det", "kvcache", "blhd", torch.bfloat16, B=6, Lq=4, Hq=32, Hkv=4, Lk=2000, Dqk=128,
                    Dv=128, causal=True, seed=3, seqlen_lo=1, seqlen_hi=2000)
    q, k, v, sl = wl.make_inputs(w, DEV)
    a = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=True)
    b = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_automatic_choice():
    """The library's own choice: 8-row blocks while the re-reads they cost
    stay small, the tcgen05 split-KV kernel from 128 MB of saved re-reads."""
    fa.force_variant(fa.VARIANT_AUTO)
    for (B, Lk, Hkv, g, lq), want in (((1, 128, 2, 4, 32), fa.VARIANT_MMA),       # 64 KB of K/V (C1's shape)
                                      ((1, 8192, 8, 8, 4), fa.VARIANT_MMA),       # 33.5 MB, 3x re-read
                                      ((4, 8192, 8, 8, 4), fa.VARIANT_TCGEN05_SPLIT),  # 134 MB, 3x re-read
                                      ((1, 8192, 8, 8, 1), fa.VARIANT_MMA)):      # 8 rows: one block
        q = torch.zeros(B, lq, g * Hkv, 128, dtype=torch.bfloat16, device=DEV)
        k = torch.zeros(B, Lk, Hkv, 128, dtype=torch.bfloat16, device=DEV)
        fa.fa_fwd(q, k, k, causal=True)
        torch.cuda.synchronize()
        assert fa.last_dispatch()["variant"] == want, (B, Lk, Hkv, g, lq, fa.last_dispatch())


@pytest.mark.slow
def test_gqa8_specdec_kvcache_full_size_sampled():
    """The batched GQA-8 speculative decode (B64, qLen 4, Hq 64 / Hkv 8, D128,
    cache lengths U[1, 16384]) in the bench's launch configuration, on
    sampled rows."""
    fa.force_variant(fa.VARIANT_AUTO)  # the library's own choice at this size
    w = wl.WORKLOADS["gqa8_specdec_kvcache_bf16"]
    q, k, v, sl = wl.make_inputs(w, DEV)
    o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=w.causal)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    assert d["variant"] == fa.VARIANT_TCGEN05_SPLIT and d["rows_per_cta"] == 32
    rows = sample_rows(w.B, w.Hq, w.Lq, 64, seed=8)
    eo, el = oracle_sampled(q, k, v, w.causal, rows, seqlens=sl)
    go, gl = gather_rows(o, lse, rows)
    compare(go, gl, eo, el, w.dtype, "gqa8 specdec full")
