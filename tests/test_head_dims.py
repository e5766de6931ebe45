"""GPU parity of head dims other than the compiled kernels' (any multiple of 8
from 8 to 256, Dqk and Dv independent) through every entry point of the C ABI:
each call runs on the instance whose dims cover it, the extra dims read as
zeros and never written (the output's row stride equals the call's Dv, so a
write past it would land in the next head's row and fail the comparison)."""
import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import compare, lse_to_numpy, o_to_numpy, oracle_full

pytestmark = pytest.mark.gpu

DEV = "cuda"
DIMS = [(8, 8), (32, 32), (40, 40), (72, 72), (80, 80), (96, 96), (112, 112), (160, 160), (200, 200), (248, 248),
        (64, 128), (128, 64), (160, 128), (136, 96), (256, 96), (96, 256)]


@pytest.fixture(autouse=True)
def _reset():
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


def _dt(i):
    return torch.float16 if i % 2 == 0 else torch.bfloat16


@pytest.mark.parametrize("i,d", list(enumerate(DIMS)), ids=[f"{a}x{b}" for a, b in DIMS])
def test_dense(i, d):
    dt = _dt(i)
    causal = i % 3 != 0
    w = wl.Workload("hd", "fwd", "blhd", dt, B=2, Lq=[1, 3, 8][i % 3], Hq=[2, 8, 12][i % 3], Hkv=[2, 2, 3][i % 3],
                    Lk=[333, 1000, 129][i % 3], Dqk=d[0], Dv=d[1], causal=causal, seed=500 + i)
    q, k, v, _ = wl.make_inputs(w, DEV)
    o, lse = fa.fa_fwd(q, k, v, causal=causal, num_splits=[0, 1, 5][i % 3])
    torch.cuda.synchronize()
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, f"dense {d}")


@pytest.mark.parametrize("i,d", list(enumerate(DIMS[::3])), ids=[f"{a}x{b}" for a, b in DIMS[::3]])
def test_kvcache(i, d):
    dt = _dt(i + 1)
    w = wl.Workload("hd_kv", "kvcache", "blhd", dt, B=5, Lq=2, Hq=8, Hkv=2, Lk=900, Dqk=d[0], Dv=d[1], causal=True,
                    seed=600 + i, seqlen_lo=0, seqlen_hi=900)
    q, k, v, sl = wl.make_inputs(w, DEV)
    o, lse = fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle_full(q, k, v, True, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, f"kvcache {d}")


@pytest.mark.parametrize("d", [(80, 80), (160, 128), (40, 40)])
def test_paged(d):
    w = wl.Workload("hd_pg", "paged", "blhd", torch.bfloat16, B=3, Lq=1, Hq=4, Hkv=4, Lk=700, Dqk=d[0], Dv=d[1],
                    causal=False, seed=700 + d[0], seqlen_lo=0, seqlen_hi=700, page=32)
    q, kp, vp, bt, sl = wl.make_paged_inputs(w, DEV, poison=True)
    o, lse = fa.fa_decode_kvcache_paged(q, kp, vp, bt, sl.to(DEV))
    torch.cuda.synchronize()
    ro, rl = oracle.attention_paged(q.cpu(), kp.cpu(), vp.cpu(), bt.cpu().numpy(), sl.numpy(), causal=False)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, f"paged {d}")


@pytest.mark.parametrize("d", [(96, 96), (200, 200)])
def test_varlen(d):
    lq, lk = [1, 4, 2], [300, 1025, 0]
    g = torch.Generator(device=DEV).manual_seed(d[0])
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    q = torch.randn(int(cq[-1]), 8, d[0], generator=g, device=DEV).half()
    k = torch.randn(int(ck[-1]), 2, d[0], generator=g, device=DEV).half()
    v = torch.randn(int(ck[-1]), 2, d[1], generator=g, device=DEV).half()
    o, lse = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), max(lq), max(lk), causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_varlen(q.cpu(), k.cpu(), v.cpu(), cq.numpy(), ck.numpy(), causal=True)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, torch.float16, f"varlen {d}")


@pytest.mark.parametrize("d", [(72, 72), (128, 64)])
def test_append(d):
    w = wl.Workload("hd_app", "kvcache", "blhd", torch.bfloat16, B=3, Lq=2, Hq=4, Hkv=2, Lk=400, Dqk=d[0], Dv=d[1],
                    causal=True, seed=800 + d[0], seqlen_lo=0, seqlen_hi=398)
    q, kc, vc, sl = wl.make_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(9)
    kn = torch.randn(3, 2, 2, d[0], generator=g, device=DEV).bfloat16()
    vn = torch.randn(3, 2, 2, d[1], generator=g, device=DEV).bfloat16()
    want_k, want_v = oracle.append_kv(kc.cpu(), vc.cpu(), kn.cpu(), vn.cpu(), sl.numpy())
    o, lse = fa.fa_decode_kvcache_append(q, kn, vn, kc, vc, sl.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu(), want_k) and torch.equal(vc.cpu(), want_v)
    ro, rl = oracle.attention(q.cpu(), want_k, want_v, causal=True, seqlens=sl.numpy() + 2)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, f"append {d}")


@pytest.mark.parametrize("d", [(80, 80), (48, 48), (160, 128)])
def test_scalar_variant(d):
    w = wl.Workload("hd_sc", "fwd", "blhd", torch.float16, B=2, Lq=1, Hq=3, Hkv=3, Lk=2000, Dqk=d[0], Dv=d[1],
                    causal=False, seed=900 + d[0])
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_SCALAR)
    o, lse = fa.fa_fwd(q, k, v)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_SCALAR
    ro, rl = oracle_full(q, k, v, False)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, torch.float16, f"scalar {d}")


def test_prefill_shaped_call_on_the_split_kernel():
    # 256 packed rows with head dim 96: not a tcgen05 prefill shape, the split-KV kernel takes it
    # (8-row blocks at this size; forced, the tcgen05 split-KV kernel's row blocks of 64)
    w = wl.Workload("hd_pf", "fwd", "blhd", torch.bfloat16, B=1, Lq=64, Hq=8, Hkv=2, Lk=500, Dqk=96, Dv=96,
                    causal=True, seed=77)
    q, k, v, _ = wl.make_inputs(w, DEV)
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_MMA
    ro, rl = oracle_full(q, k, v, True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, torch.bfloat16, "prefill-shaped hd 96")
    fa.force_variant(fa.VARIANT_TCGEN05_SPLIT)  # and on the tcgen05 split-KV kernel's 64-row blocks
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["rows_per_cta"] == 64
    fa.force_variant(fa.VARIANT_AUTO)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, torch.bfloat16, "prefill-shaped hd 96, tcgen05 split")


def test_instance_dims_in_dispatch():
    for (dqk, dv), want_smem_same_as in (((80, 80), (128, 128)), ((40, 40), (64, 64)), ((160, 128), (192, 128))):
        qs = [torch.zeros(1, 1, 4, d0, dtype=torch.float16, device=DEV) for d0 in (dqk, want_smem_same_as[0])]
        res = []
        for qq, (a, b) in zip(qs, ((dqk, dv), want_smem_same_as)):
            k = torch.zeros(1, 64, 4, a, dtype=torch.float16, device=DEV)
            v = torch.zeros(1, 64, 4, b, dtype=torch.float16, device=DEV)
            fa.fa_fwd(qq, k, v)
            res.append(fa.last_dispatch()["smem_bytes"])
        assert res[0] == res[1], ((dqk, dv), res)
