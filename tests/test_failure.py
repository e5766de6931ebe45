"""The failure path on the GPU, made without a fault: a test hook leaves one
pipeline stage of the split-KV kernel empty (a barrier phase nothing
completes) and bounds the call's waits by 20 ms.  The waiting warps give up,
record FA_ERR_TIMEOUT in the device status word and return; the host reads it
with check_status, and the next call on the same context runs normally and
matches the oracle.  Covered for the mma.sync kernel, its fp32 FMA form, the
tcgen05 split-KV kernel and both forms of the tcgen05 prefill kernel (whose
abort paths must also wait for their tensor-core work and free their tensor
memory before the next call can allocate it)."""
import time

import pytest
import torch

import decode_flashattention_b200 as fa
from decode_flashattention_b200 import workloads as wl

from helpers import compare, lse_to_numpy, o_to_numpy, oracle_full

pytestmark = pytest.mark.gpu

DEV = "cuda"
FA_ERR_TIMEOUT = 5
LIMIT_NS = 20_000_000  # 20 ms


@pytest.fixture(autouse=True)
def _reset():
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    fa.force_tcgen05_form(fa.TCGEN05_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


def _call(variant, w, q, k, v, sl):
    fa.force_variant(variant)
    if sl is None:
        return fa.fa_fwd(q, k, v, causal=w.causal)
    return fa.fa_decode_kvcache(q, k, v, sl.to(DEV), causal=w.causal)


@pytest.mark.parametrize("variant", [fa.VARIANT_MMA, fa.VARIANT_SCALAR, fa.VARIANT_TCGEN05_SPLIT])
def test_timeout_is_reported_and_the_context_stays_usable(variant):
    if variant == fa.VARIANT_SCALAR:  # one packed row
        w = wl.Workload("stall_sc", "fwd", "blhd", torch.float16, B=1, Lq=1, Hq=4, Hkv=4, Lk=3000, Dqk=128, Dv=128,
                        causal=False, seed=31)
    elif variant == fa.VARIANT_TCGEN05_SPLIT:  # 16 packed rows per kv head
        w = wl.Workload("stall_tc", "kvcache", "blhd", torch.bfloat16, B=6, Lq=4, Hq=8, Hkv=2, Lk=3000, Dqk=128,
                        Dv=128, causal=True, seed=33, seqlen_lo=1, seqlen_hi=3000)
    else:
        w = wl.Workload("stall_kv", "kvcache", "blhd", torch.bfloat16, B=6, Lq=2, Hq=8, Hkv=2, Lk=3000, Dqk=128,
                        Dv=128, causal=True, seed=32, seqlen_lo=1, seqlen_hi=3000)
    q, k, v, sl = wl.make_inputs(w, DEV)
    fa.check_status()  # nothing pending
    fa.test_stall_next_call(LIMIT_NS)
    t0 = time.perf_counter()
    _call(variant, w, q, k, v, sl)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    with pytest.raises(fa.FaError) as e:
        fa.check_status()
    assert e.value.status == FA_ERR_TIMEOUT
    assert elapsed < 2.0, elapsed  # the 20 ms bound was used, not the 4 s default
    fa.check_status()  # reading the timeout cleared it
    # the same context runs the next call normally
    o, lse = _call(variant, w, q, k, v, sl)
    torch.cuda.synchronize()
    fa.check_status()
    ro, rl = oracle_full(q, k, v, w.causal, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "after a timeout")


@pytest.mark.parametrize("form", [fa.TCGEN05_TWO_TILES, fa.TCGEN05_ONE_TILE_MMA])
def test_prefill_timeout_is_reported_and_the_context_stays_usable(form):
    # 512 packed rows per kv head (two or four row blocks), causal, ragged keys:
    # the stalled CTA (the grid's first, the last row block) has tiles to wait for
    w = wl.Workload("stall_pf", "fwd", "blhd", torch.bfloat16, B=1, Lq=256, Hq=4, Hkv=2, Lk=700, Dqk=128, Dv=128,
                    causal=True, seed=34)
    q, k, v, _ = wl.make_inputs(w, DEV)

    def call():
        fa.force_variant(fa.VARIANT_TCGEN05)
        fa.force_tcgen05_form(form)
        return fa.fa_fwd(q, k, v, causal=True)

    fa.check_status()
    fa.test_stall_next_call(LIMIT_NS)
    t0 = time.perf_counter()
    call()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert fa.last_dispatch()["tcgen05_form"] == form
    with pytest.raises(fa.FaError) as e:
        fa.check_status()
    assert e.value.status == FA_ERR_TIMEOUT
    assert elapsed < 2.0, elapsed
    fa.check_status()
    o, lse = call()  # allocates the tensor memory the stalled CTA held
    torch.cuda.synchronize()
    fa.check_status()
    ro, rl = oracle_full(q, k, v, True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "prefill after a timeout")
