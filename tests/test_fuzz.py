"""Seeded random parity sweep over every entry point of the C ABI.

Each case draws a call (dense, kvcache, paged, append or varlen), head dims
(the compiled kernels' and others that run zero-padded on them),
element type, GQA ratio, query length 1-8, causal flag, split count and
variant (the library's choice, the fp32 FMA form for one packed row, or the
tcgen05 split-KV kernel for more than 8), with ragged lengths, and compares the result with the oracle
element by element.  The draws are fixed by the seed, so a failure names a
reproducible case."""
import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import compare, lse_to_numpy, o_to_numpy, oracle_full

pytestmark = pytest.mark.gpu

DEV = "cuda"
N_CASES = 100
DIMS = [(64, 64), (128, 128), (192, 128), (256, 256), (80, 80), (96, 96), (40, 40), (160, 128), (112, 112)]


def _runs_on_256(d):
    """Whether the call runs on the (256, 256) kernel, which has no fp32-FMA form."""
    return not (128 < d[0] <= 192 and d[1] <= 128) and max(d) > 128


def _draw(i):
    r = np.random.default_rng(10_000 + i)
    call = ["dense", "kvcache", "paged", "append", "varlen"][i % 5]
    d = DIMS[int(r.integers(0, len(DIMS)))]
    dt = torch.float16 if r.random() < 0.5 else torch.bfloat16
    Hkv = int(r.choice([1, 2, 3]))
    g = int(r.choice([1, 2, 4, 5, 8, 12]))
    lq = int(r.integers(1, 9))
    B = int(r.integers(1, 6))
    lk = int(r.choice([1, 7, 64, 127, 128, 129, 300, 1000, 2500]))
    causal = bool(r.random() < 0.5)
    splits = int(r.choice([0, 0, 1, 2, 9]))
    variant = fa.VARIANT_SCALAR if (g * lq == 1 and not _runs_on_256(d) and r.random() < 0.5) else fa.VARIANT_AUTO
    page = int(r.choice([16, 32, 64, 128, 256]))
    # more than 8 packed rows: half the cases forced onto the tcgen05 split-KV
    # kernel (at these sizes the library itself keeps the 8-row blocks)
    fits_tc = (d[1] <= 128 and d[0] <= 192) if not _runs_on_256(d) else False
    if g * lq > 8 and fits_tc and r.random() < 0.5:
        variant = fa.VARIANT_TCGEN05_SPLIT
    return call, d, dt, Hkv, g, lq, B, lk, causal, splits, variant, page, r


@pytest.fixture(autouse=True)
def _reset():
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


@pytest.mark.parametrize("i", range(N_CASES))
def test_fuzz(i):
    call, d, dt, Hkv, g, lq, B, lk, causal, splits, variant, page, r = _draw(i)
    fa.force_variant(variant)
    Hq = g * Hkv
    name = f"fuzz{i}:{call}"
    if call == "dense":
        w = wl.Workload(name, "fwd", "blhd", dt, B=B, Lq=lq, Hq=Hq, Hkv=Hkv, Lk=lk, Dqk=d[0], Dv=d[1],
                        causal=causal, seed=i)
        q, k, v, _ = wl.make_inputs(w, DEV)
        o, lse = fa.fa_fwd(q, k, v, causal=causal, num_splits=splits)
        torch.cuda.synchronize()
        ro, rl = oracle_full(q, k, v, causal)
    elif call in ("kvcache", "append"):
        w = wl.Workload(name, "kvcache", "blhd", dt, B=B, Lq=lq, Hq=Hq, Hkv=Hkv, Lk=lk, Dqk=d[0], Dv=d[1],
                        causal=causal, seed=i, seqlen_lo=0, seqlen_hi=lk)
        q, k, v, sl = wl.make_inputs(w, DEV)
        if call == "kvcache":
            o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=causal, num_splits=splits)
            torch.cuda.synchronize()
            ro, rl = oracle_full(q, k, v, causal, seqlens=sl)
        else:
            kn = torch.randn(B, lq, Hkv, d[0], device=DEV).to(dt)
            vn = torch.randn(B, lq, Hkv, d[1], device=DEV).to(dt)
            want_k, want_v = oracle.append_kv(k.cpu(), v.cpu(), kn.cpu(), vn.cpu(), sl.numpy())
            o, lse = fa.fa_decode_kvcache_append(q, kn, vn, k, v, sl.to(DEV), causal=causal, num_splits=splits)
            torch.cuda.synchronize()
            assert torch.equal(k.cpu(), want_k) and torch.equal(v.cpu(), want_v)
            n = np.minimum(sl.numpy() + lq, lk)
            ro, rl = oracle.attention(q.cpu(), want_k, want_v, causal=causal, seqlens=n)
    elif call == "paged":
        w = wl.Workload(name, "paged", "blhd", dt, B=B, Lq=lq, Hq=Hq, Hkv=Hkv, Lk=lk, Dqk=d[0], Dv=d[1],
                        causal=causal, seed=i, seqlen_lo=0, seqlen_hi=lk, page=page)
        q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV, poison=True)
        o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV), causal=causal, num_splits=splits)
        torch.cuda.synchronize()
        ro, rl = oracle.attention_paged(q.cpu(), kp.cpu(), vp.cpu(), bt.cpu().numpy(), sl.numpy(), causal=causal)
    else:  # varlen
        lqs = [int(x) for x in r.integers(0, lq + 1, B)]
        lks = [int(x) for x in r.integers(0, lk + 1, B)]
        cq = torch.tensor(np.concatenate([[0], np.cumsum(lqs)]), dtype=torch.int32)
        ck = torch.tensor(np.concatenate([[0], np.cumsum(lks)]), dtype=torch.int32)
        gen = torch.Generator(device=DEV).manual_seed(i)
        q = torch.randn(int(cq[-1]), Hq, d[0], generator=gen, device=DEV).to(dt)
        k = torch.randn(max(int(ck[-1]), 1), Hkv, d[0], generator=gen, device=DEV).to(dt)
        v = torch.randn(max(int(ck[-1]), 1), Hkv, d[1], generator=gen, device=DEV).to(dt)
        if int(cq[-1]) == 0:
            pytest.skip("no query tokens drawn")
        o, lse = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), max(max(lqs), 1), max(max(lks), 1),
                                  causal=causal, num_splits=splits)
        torch.cuda.synchronize()
        ro, rl = oracle.attention_varlen(q.cpu(), k.cpu(), v.cpu(), cq.numpy(), ck.numpy(), causal=causal)
        compare(o.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, dt, name)
        return
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, name)
