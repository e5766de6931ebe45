"""GPU parity of the tcgen05 kernels (dense fa_fwd with >= 128 packed rows,
head dims 128/128, and 64/64 in the two-tile kernel's forms) against the
oracle: ragged query and key lengths, causal bottom-right alignment
including rows with no visible key, GQA packing, fp16 / bf16, several
batches; full-size prefill on sampled rows."""
import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle
from decode_flashattention_b200 import workloads as wl

from helpers import compare, o_to_numpy, lse_to_numpy, oracle_full

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _reset():
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    fa.force_tcgen05_form(fa.TCGEN05_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


FORMS = [fa.TCGEN05_TWO_TILES, fa.TCGEN05_ONE_TILE_MMA]


CASES = [  # B, Lq, Hq, Hkv, Lk, causal
    (1, 128, 1, 1, 128, False), (1, 129, 1, 1, 1, False), (2, 300, 2, 1, 700, True), (1, 1000, 4, 4, 1000, True),
    (3, 64, 8, 4, 257, False), (1, 32, 8, 2, 128, True), (1, 1, 128, 1, 3000, False), (1, 500, 2, 2, 200, True),
    (1, 257, 16, 2, 129, True), (2, 160, 4, 1, 4000, False),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_tcgen05_parity(case, dt):
    B, Lq, Hq, Hkv, Lk, causal = case
    w = wl.Workload("pf", "fwd", "blhd", dt, B=B, Lq=Lq, Hq=Hq, Hkv=Hkv, Lk=Lk, Dqk=128, Dv=128, causal=causal,
                    seed=Lq + Lk)
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_TCGEN05)  # small calls would otherwise go to the split-KV kernel
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, "tcgen05")


def test_forced_on_fewer_rows_and_refused_for_caches():
    w = wl.Workload("pf2", "fwd", "blhd", torch.bfloat16, B=2, Lq=3, Hq=2, Hkv=2, Lk=300, Dqk=128, Dv=128,
                    causal=True, seed=4)
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_TCGEN05)
    o, lse = fa.fa_fwd(q, k, v, causal=True)  # 6 rows in a 128-row tile: the rest is padding
    torch.cuda.synchronize()
    ro, rl = oracle_full(q, k, v, True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, torch.bfloat16, "tcgen05 forced")
    sl = torch.tensor([10, 300], dtype=torch.int32, device=DEV)
    with pytest.raises(fa.FaError, match="tcgen05"):
        fa.fa_decode_kvcache(q, k, v, sl)


def test_full_size_prefill_sampled_rows():
    w = wl.WORKLOADS["gqa_prefill4k_bf16"]
    q, k, v, _ = wl.make_inputs(w, DEV)
    o, lse = fa.fa_fwd(q, k, v, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05
    rng = np.random.default_rng(0)
    rows = np.stack([rng.integers(0, w.B, 48), rng.integers(0, w.Hq, 48), rng.integers(0, w.Lq, 48)], 1)
    ro, rl = oracle.attention(q.cpu(), k.cpu(), v.cpu(), causal=w.causal, rows=rows)
    got_o = o.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_l = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    compare(got_o, got_l, ro, rl, w.dtype, "prefill 4k")


FORM_CASES = [  # B, Lq, Hq, Hkv, Lk, causal: ragged row blocks (R % 256 below and above 128), short and long keys
    (1, 200, 2, 1, 300, True), (2, 130, 4, 2, 129, False), (1, 700, 1, 1, 700, True), (3, 96, 8, 2, 1000, True),
    (1, 64, 32, 8, 2500, False), (1, 1, 256, 1, 77, False),
    (1, 300, 2, 1, 100, True),  # causal with Lq > Lk: the first 200 positions see no key
]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("case", FORM_CASES, ids=[str(c) for c in FORM_CASES])
def test_every_form_parity(form, case):
    B, Lq, Hq, Hkv, Lk, causal = case
    dt = torch.bfloat16 if (Lq + form) % 2 else torch.float16
    w = wl.Workload("pf_form", "fwd", "blhd", dt, B=B, Lq=Lq, Hq=Hq, Hkv=Hkv, Lk=Lk, Dqk=128, Dv=128, causal=causal,
                    seed=Lq * 7 + Lk + form)
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_TCGEN05)
    fa.force_tcgen05_form(form)
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    assert d["variant"] == fa.VARIANT_TCGEN05 and d["tcgen05_form"] == form
    assert d["rows_per_cta"] == (256 if form == fa.TCGEN05_TWO_TILES else 128)
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, f"tcgen05 form {form}")


def test_automatic_kernel_and_form_choice():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for (B, Lq, Hq, Hkv, D), (var, form) in (
            ((1, 4096, 32, 8, 128), (fa.VARIANT_TCGEN05, fa.TCGEN05_TWO_TILES)),   # 64 x 8 two-tile CTAs
            ((1, 300, 16, 16, 128), (fa.VARIANT_TCGEN05, fa.TCGEN05_ONE_TILE_MMA)),  # 2 x 16 two-tile CTAs
            ((4, 32, 32, 8, 128), (fa.VARIANT_TCGEN05, fa.TCGEN05_ONE_TILE_MMA)),  # 128 rows, 32 CTAs
            ((4, 32, 32, 8, 64), (fa.VARIANT_TCGEN05, fa.TCGEN05_ONE_TILE_MMA)),   # the same with 64-dim heads
            ((1, 300, 16, 16, 64), (fa.VARIANT_TCGEN05, fa.TCGEN05_ONE_TILE_MMA)), # 64-dim heads: no serial form
            ((2, 32, 32, 8, 128), (fa.VARIANT_MMA, 0)),                            # 16 CTAs: split-KV kernel
            ((1, 32, 8, 2, 64), (fa.VARIANT_MMA, 0))):                             # 2 CTAs (the 64-key prefill)
        if form == fa.TCGEN05_TWO_TILES:
            assert ((Lq * Hq // Hkv + 255) // 256) * Hkv * B >= sms
        q = torch.zeros(B, Lq, Hq, D, dtype=torch.bfloat16, device=DEV)
        k = torch.zeros(B, 256, Hkv, D, dtype=torch.bfloat16, device=DEV)
        fa.fa_fwd(q, k, k, causal=True)
        torch.cuda.synchronize()
        d = fa.last_dispatch()
        assert (d["variant"], d["tcgen05_form"]) == (var, form), ((B, Lq, Hq, Hkv, D), d)


HD64_CASES = [  # B, Lq, Hq, Hkv, Lk, causal
    (1, 200, 2, 1, 300, True), (2, 130, 4, 2, 129, False), (1, 32, 8, 2, 128, True), (1, 300, 2, 1, 100, True),
    (1, 1000, 4, 4, 2000, True),
]


@pytest.mark.parametrize("form", [fa.TCGEN05_TWO_TILES, fa.TCGEN05_ONE_TILE_MMA])
@pytest.mark.parametrize("case", HD64_CASES, ids=[str(c) for c in HD64_CASES])
def test_head_dim_64_parity(form, case):
    B, Lq, Hq, Hkv, Lk, causal = case
    dt = torch.float16 if (Lq + form) % 2 else torch.bfloat16
    w = wl.Workload("pf64", "fwd", "blhd", dt, B=B, Lq=Lq, Hq=Hq, Hkv=Hkv, Lk=Lk, Dqk=64, Dv=64, causal=causal,
                    seed=Lq + Lk + 64 * form)
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_TCGEN05)
    fa.force_tcgen05_form(form)
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    assert d["variant"] == fa.VARIANT_TCGEN05 and d["tcgen05_form"] == form
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, f"tcgen05 hd64 form {form}")




MLA_CASES = [  # B, Lq, Hq, Hkv, Lk, causal
    (1, 200, 2, 1, 300, True), (2, 130, 4, 2, 129, False), (1, 300, 2, 1, 100, True), (1, 1000, 4, 4, 1000, True),
    (1, 64, 8, 2, 700, False),
]


@pytest.mark.parametrize("form", [fa.TCGEN05_TWO_TILES, fa.TCGEN05_ONE_TILE_MMA])
@pytest.mark.parametrize("case", MLA_CASES, ids=[str(c) for c in MLA_CASES])
def test_mla_head_dims_parity(form, case):
    """Head dims 192 / 128 (Q and K rows of three 64-column boxes, V rows of
    two; K and V take turns in two ring slots)."""
    B, Lq, Hq, Hkv, Lk, causal = case
    dt = torch.float16 if (Lq + form) % 2 else torch.bfloat16
    w = wl.Workload("pf192", "fwd", "blhd", dt, B=B, Lq=Lq, Hq=Hq, Hkv=Hkv, Lk=Lk, Dqk=192, Dv=128, causal=causal,
                    seed=Lq + Lk + 192 * form)
    q, k, v, _ = wl.make_inputs(w, DEV)
    fa.force_variant(fa.VARIANT_TCGEN05)
    fa.force_tcgen05_form(form)
    o, lse = fa.fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    assert d["variant"] == fa.VARIANT_TCGEN05 and d["tcgen05_form"] == form
    ro, rl = oracle_full(q, k, v, causal)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, dt, f"tcgen05 192/128 form {form}")


def test_mla_head_dims_automatic_choice():
    """A large prefill-shaped call with head dims 192 / 128 runs on the dense
    tcgen05 kernel; other non-square dims stay on the split-KV kernels."""
    q = torch.zeros(1, 2048, 32, 192, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 512, 8, 192, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(1, 512, 8, 128, dtype=torch.bfloat16, device=DEV)
    fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    d = fa.last_dispatch()
    assert (d["variant"], d["tcgen05_form"]) == (fa.VARIANT_TCGEN05, fa.TCGEN05_TWO_TILES), d
    q2 = torch.zeros(1, 2048, 32, 160, dtype=torch.bfloat16, device=DEV)
    k2 = torch.zeros(1, 512, 8, 160, dtype=torch.bfloat16, device=DEV)
    fa.fa_fwd(q2, k2, v, causal=True)
    torch.cuda.synchronize()
    assert fa.last_dispatch()["variant"] == fa.VARIANT_TCGEN05_SPLIT
