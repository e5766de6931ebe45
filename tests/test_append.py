"""GPU parity of fa_decode_kvcache_append (through the C ABI): the cache after
the call equals the oracle's append bit for bit, and the output equals the
oracle's attention over cache_seqlens[b] + Lnew keys; dense and paged caches,
one or several new tokens, causal and not, lengths at the capacity edge."""
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
def _status():
    yield
    torch.cuda.synchronize()
    fa.check_status()


def _new(B, Lnew, Hkv, d, dt, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    kn = torch.randn(B, Lnew, Hkv, d[0], generator=g, device=DEV).to(dt)
    vn = torch.randn(B, Lnew, Hkv, d[1], generator=g, device=DEV).to(dt)
    return kn, vn


@pytest.mark.parametrize("lnew,g,causal", [(1, 1, False), (1, 4, False), (4, 2, True), (8, 1, True)])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_dense_append(lnew, g, causal, dt):
    w = wl.Workload("app", "kvcache", "blhd", dt, B=4, Lq=lnew, Hq=2 * g, Hkv=2, Lk=700, Dqk=128, Dv=128,
                    causal=causal, seed=40 + lnew + g, seqlen_lo=0, seqlen_hi=700 - lnew)
    q, kc, vc, sl = wl.make_inputs(w, DEV)
    sl[0] = 0
    sl[-1] = 700 - lnew  # fills the cache exactly
    kn, vn = _new(w.B, lnew, w.Hkv, (128, 128), dt, 7)
    want_k, want_v = oracle.append_kv(kc.cpu(), vc.cpu(), kn.cpu(), vn.cpu(), sl.numpy())
    o, lse = fa.fa_decode_kvcache_append(q, kn, vn, kc, vc, sl.to(DEV), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu(), want_k) and torch.equal(vc.cpu(), want_v)
    ro, rl = oracle.attention(q.cpu(), want_k, want_v, causal=causal, seqlens=sl.numpy() + lnew)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, "append dense")


@pytest.mark.parametrize("page", [16, 64, 256])
@pytest.mark.parametrize("lnew", [1, 4])
def test_paged_append(page, lnew):
    w = wl.Workload("app_p", "paged", "blhd", torch.bfloat16, B=5, Lq=lnew, Hq=8, Hkv=2, Lk=900, Dqk=128, Dv=128,
                    causal=lnew > 1, seed=60 + page + lnew, seqlen_lo=0, seqlen_hi=890, page=page)
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV)
    # give every batch the blocks its appended tokens need (fresh ones from a grown pool)
    nb0 = kp.shape[0]
    extra = []
    for b in range(w.B):
        have = -(-int(sl[b]) // page)
        need = -(-(int(sl[b]) + lnew) // page)
        for i in range(have, need):
            bt[b, i] = nb0 + len(extra)
            extra.append(b)
    if extra:
        g = torch.Generator(device=DEV).manual_seed(5)
        kp = torch.cat([kp, torch.randn(len(extra), page, w.Hkv, 128, generator=g, device=DEV).to(kp.dtype)])
        vp = torch.cat([vp, torch.randn(len(extra), page, w.Hkv, 128, generator=g, device=DEV).to(vp.dtype)])
    kn, vn = _new(w.B, lnew, w.Hkv, (128, 128), torch.bfloat16, 9)
    btn = bt.cpu().numpy()
    want_k, want_v = oracle.append_kv(kp.cpu(), vp.cpu(), kn.cpu(), vn.cpu(), sl.numpy(), block_table=btn)
    o, lse = fa.fa_decode_kvcache_append(q, kn, vn, kp, vp, sl.to(DEV), block_table=bt, causal=w.causal)
    torch.cuda.synchronize()
    assert torch.equal(kp.cpu(), want_k) and torch.equal(vp.cpu(), want_v)
    ro, rl = oracle.attention_paged(q.cpu(), want_k, want_v, btn, sl.numpy() + lnew, causal=w.causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "append paged")


def test_flash_attn_with_kvcache_appends():
    w = wl.Workload("app2", "kvcache", "blhd", torch.float16, B=2, Lq=1, Hq=4, Hkv=4, Lk=300, Dqk=64, Dv=64,
                    causal=False, seed=3, seqlen_lo=10, seqlen_hi=200)
    q, kc, vc, sl = wl.make_inputs(w, DEV)
    kn, vn = _new(2, 1, 4, (64, 64), torch.float16, 1)
    kc2, vc2 = kc.clone(), vc.clone()
    o1 = fa.flash_attn_with_kvcache(q, kc, vc, sl.to(DEV), k=kn, v=vn)
    # the same as writing the token by hand and calling without append
    for b in range(2):
        kc2[b, int(sl[b])] = kn[b, 0]
        vc2[b, int(sl[b])] = vn[b, 0]
    o2 = fa.flash_attn_with_kvcache(q, kc2, vc2, (sl + 1).to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(kc, kc2) and torch.equal(o1, o2)
