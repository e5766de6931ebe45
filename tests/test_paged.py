"""GPU parity of fa_decode_kvcache_paged (through the C ABI) against the oracle.

Block tables are shuffled pools (blocks in random order, entries past a
batch's blocks set to -1), unused pool rows hold NaN, lengths are ragged
(0, 1, page and tile edges); page sizes 16 to 512 cover both ways a 128-key
tile meets the pages (several pages per tile, several tiles per page).
"""
import dataclasses

import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import compare, lse_to_numpy, o_to_numpy

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _auto_variant():
    fa.force_variant(fa.VARIANT_AUTO)
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


def _case(page, B=4, Lq=1, Hq=8, Hkv=2, Lk=1000, d=(128, 128), dt=torch.bfloat16, causal=False, seed=0,
          seqlens=None):
    w = wl.Workload("paged_t", "paged", "blhd", dt, B=B, Lq=Lq, Hq=Hq, Hkv=Hkv, Lk=Lk, Dqk=d[0], Dv=d[1],
                    causal=causal, seed=seed, seqlen_lo=0, seqlen_hi=Lk, page=page)
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV, poison=True)
    if seqlens is not None:
        # rebuild the table for the given lengths from the same pool
        sl = torch.tensor(seqlens, dtype=torch.int32)
        mb = bt.shape[1]
        need = [-(-int(n) // page) for n in sl]
        assert sum(need) <= kp.shape[0]
        perm = torch.randperm(kp.shape[0], generator=torch.Generator().manual_seed(seed + 7))
        table = torch.full((B, mb), -1, dtype=torch.int32)
        pos = 0
        for b in range(B):
            table[b, :need[b]] = perm[pos:pos + need[b]].to(torch.int32)
            pos += need[b]
        bt = table.to(DEV)
        # fresh values, poisoned where the new table addresses nothing
        g = torch.Generator(device=DEV).manual_seed(seed + 9)
        kp = torch.randn(kp.shape, generator=g, device=DEV).to(dt)
        vp = torch.randn(vp.shape, generator=g, device=DEV).to(dt)
        live = torch.zeros(kp.shape[0], page, dtype=torch.bool)
        for b in range(B):
            for j0 in range(0, int(sl[b]), page):
                live[int(table[b, j0 // page]), :min(page, int(sl[b]) - j0)] = True
        kp[(~live).to(DEV)] = float("nan")
        vp[(~live).to(DEV)] = float("nan")
    return w, q, kp, vp, bt, sl


def _check(w, q, kp, vp, bt, sl, num_splits=0):
    o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV), causal=w.causal, num_splits=num_splits)
    torch.cuda.synchronize()
    fa.check_status()
    ro, rl = oracle.attention_paged(q.cpu(), kp.cpu(), vp.cpu(), bt.cpu().numpy(), sl.numpy(), causal=w.causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, f"paged{w.page}")
    return fa.last_dispatch()


@pytest.mark.parametrize("page", [16, 32, 64, 128, 256, 512])
def test_page_sizes(page):
    _check(*_case(page, seed=page))


@pytest.mark.parametrize("d", [(64, 64), (128, 128), (192, 128)])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_head_dims_and_types(d, dt):
    _check(*_case(32, d=d, dt=dt, seed=d[0] + (dt == torch.float16)))


@pytest.mark.parametrize("page,d", [(16, (256, 256)), (32, (256, 256)), (16, (64, 64)), (16, (192, 128)),
                                    (16, (96, 96)), (32, (40, 40)), (16, (128, 64))])
def test_pages_below_the_tile_every_head_dim(page, d):
    """Pages smaller than the tile: one 5-D box per page where the head dims
    are the kernel instance's own (whole 64-column chunks; the 64-key tiles
    of head dim 256 included), one box per page and chunk otherwise."""
    _check(*_case(page, d=d, Lk=700, seed=page + d[0] + d[1]))


@pytest.mark.parametrize("page", [16, 32, 64])
def test_small_pages_equal_dense_call_bitwise(page):
    """Pages gathered one 5-D box per page land the keys where the dense
    call's boxes put them: the same arithmetic, the same bits."""
    w, q, kp, vp, bt, sl = _case(page, B=3, Lk=640, seed=13 + page)
    k = oracle.gather_pages(kp.cpu(), bt.cpu().numpy(), sl.numpy()).to(DEV)
    v = oracle.gather_pages(vp.cpu(), bt.cpu().numpy(), sl.numpy()).to(DEV)
    o1, l1 = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV))
    o2, l2 = fa.fa_decode_kvcache(q, k, v, sl.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("g,lq", [(1, 1), (4, 1), (8, 1), (2, 4), (1, 8)])
def test_gqa_and_small_q_causal(g, lq):
    _check(*_case(64, Lq=lq, Hq=2 * g, Hkv=2, causal=True, seed=10 * g + lq))


def test_edge_lengths():
    lens = [0, 1, 15, 16, 17, 127, 128, 129]
    _check(*_case(16, B=len(lens), seqlens=lens, Lk=200, seed=3))


@pytest.mark.parametrize("num_splits", [1, 2, 7, 100])
def test_split_counts(num_splits):
    _check(*_case(16, Lk=3000, seed=5), num_splits=num_splits)


def test_shared_blocks_and_fma_variant():
    """Two batches pointing at the same blocks read the same keys; the FMA
    variant (one packed row) reads pages the same way."""
    w, q, kp, vp, bt, sl = _case(64, B=2, Hq=2, Hkv=2, Lk=500, seqlens=[300, 300], seed=9)
    bt[1] = bt[0]
    q[1] = q[0]
    for variant in (fa.VARIANT_MMA, fa.VARIANT_SCALAR):
        fa.force_variant(variant)
        _check(w, q, kp, vp, bt, sl)
        o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(o[0], o[1]) and torch.equal(lse[0], lse[1])


def test_paged_equals_dense_call_bitwise():
    """Same keys in the same order: the paged call and the dense kvcache call
    run the same arithmetic."""
    w, q, kp, vp, bt, sl = _case(128, B=3, Lk=640, seed=11)
    k = oracle.gather_pages(kp.cpu(), bt.cpu().numpy(), sl.numpy()).to(DEV)
    v = oracle.gather_pages(vp.cpu(), bt.cpu().numpy(), sl.numpy()).to(DEV)
    o1, l1 = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV))
    o2, l2 = fa.fa_decode_kvcache(q, k, v, sl.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_rejects_bad_pages():
    w, q, kp, vp, bt, sl = _case(16, seed=1)
    with pytest.raises(fa.FaError, match="page size"):
        fa.fa_decode_kvcache_paged(q, kp[:, :12], vp[:, :12], bt, sl.to(DEV))
    with pytest.raises(ValueError):
        fa.fa_decode_kvcache_paged(q, kp, vp, bt.t(), sl.to(DEV))


def test_full_size_paged16_sampled_rows():
    """The 16-key-page workload at full size, checked on sampled rows."""
    w = wl.WORKLOADS["gqa_paged16_bf16"]
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV)
    o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV))
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    bsub = rng.choice(w.B, 8, replace=False)
    rows = np.stack([rng.choice(bsub, 64), rng.integers(0, w.Hq, 64), np.zeros(64, dtype=np.int64)], 1)
    # gather only the sampled batches' keys on the host
    bsel = sorted(set(rows[:, 0].tolist()))
    ro, rl = oracle.attention_paged(q[bsel].cpu(), kp.cpu(), vp.cpu(), bt[bsel].cpu().numpy(),
                                    sl[bsel].numpy(),
                                    rows=np.stack([[bsel.index(b), h, i] for b, h, i in rows]))
    got_o = o.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_l = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    compare(got_o, got_l, ro, rl, w.dtype, "paged16 full")
