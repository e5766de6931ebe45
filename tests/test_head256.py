"""Head dim 256 (the SmallQ README's validation shapes include hd 256): the
split-KV kernel runs 64-key tiles for it; parity against the oracle for the
dense, kvcache, paged and append calls, with GQA, causal small-Q, ragged
lengths and split counts."""
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import compare, lse_to_numpy, o_to_numpy, oracle_full

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _status():
    yield
    torch.cuda.synchronize()
    fa.check_status()


@pytest.mark.parametrize("kv,lq,g,causal,dt", [(1, 1, 1, False, torch.float16), (63, 4, 2, True, torch.bfloat16),
                                               (64, 1, 8, False, torch.float16), (65, 8, 1, True, torch.float16),
                                               (3000, 2, 4, True, torch.bfloat16), (4096, 1, 1, False, torch.float16)])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_fwd_d256(kv, lq, g, causal, dt, num_splits):
    w = wl.Workload("d256", "fwd", "blhd", dt, B=2, Lq=lq, Hq=2 * g, Hkv=2, Lk=kv, Dqk=256, Dv=256,
                    causal=causal, seed=kv + lq)
    q, k, v, _ = wl.make_inputs(w, DEV)
    o, lse = fa.fa_fwd(q, k, v, causal=causal, num_splits=num_splits)
    torch.cuda.synchronize()
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, "d256")
    assert fa.last_dispatch()["tile_keys"] == 64


def test_kvcache_d256_poisoned():
    w = wl.Workload("d256kv", "kvcache", "blhd", torch.bfloat16, B=5, Lq=1, Hq=8, Hkv=2, Lk=900, Dqk=256, Dv=256,
                    causal=False, seed=5, seqlen_lo=0, seqlen_hi=900)
    q, k, v, sl = wl.make_inputs(w, DEV)
    for b in range(w.B):
        k[b, int(sl[b]):] = float("nan")
        v[b, int(sl[b]):] = float("nan")
    o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV))
    torch.cuda.synchronize()
    ro, rl = oracle_full(q, k, v, False, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "d256 kvcache")


@pytest.mark.parametrize("page", [16, 128])
def test_paged_append_d256(page):
    w = wl.Workload("d256p", "paged", "blhd", torch.float16, B=3, Lq=2, Hq=4, Hkv=2, Lk=600, Dqk=256, Dv=256,
                    causal=True, seed=7 + page, seqlen_lo=1, seqlen_hi=590, page=page)
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV)
    o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_paged(q.cpu(), kp.cpu(), vp.cpu(), bt.cpu().numpy(), sl.numpy(), causal=True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "d256 paged")
