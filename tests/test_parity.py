"""GPU parity: the CUDA path against the fp64 oracle on identical seeded inputs.

Every call goes through the C ABI (via the ctypes binding).  Sizes the oracle
finishes in seconds are compared element by element; the full-size
workloads are compared on sampled rows the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
from decode_flashattention_b200 import workloads as wl

from helpers import (compare, gather_rows, lse_to_numpy, o_to_numpy, oracle_full, oracle_sampled,
                     sample_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _auto_variant():
    fa.force_variant(fa.VARIANT_AUTO)
    yield
    fa.force_variant(fa.VARIANT_AUTO)
    torch.cuda.synchronize()
    fa.check_status()


def run_workload(w, q, k, v, seqlens, num_splits=0, out=None):
    if out is None:
        out = wl.empty_output(w, q)
    if w.call == "kvcache":
        sl = seqlens.to(DEV)
        o, lse = fa.fa_decode_kvcache(q, k, v, sl, causal=w.causal, num_splits=num_splits, out=out)
    else:
        o, lse = fa.fa_fwd(q, k, v, causal=w.causal, num_splits=num_splits, out=out)
    torch.cuda.synchronize()
    return o, lse


def check_full(w, num_splits=0, seed=None, **over):
    w2 = w if not over else __import__("dataclasses").replace(w, **over)
    q, k, v, sl = wl.make_inputs(w2, DEV, seed=seed)
    o, lse = run_workload(w2, q, k, v, sl, num_splits)
    ro, rl = oracle_full(q, k, v, w2.causal, seqlens=sl)
    return compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w2.dtype, w2.name), fa.last_dispatch()


# ------------------------------------------------------------------ the five workloads

def test_gqa_prefill_fp16_full():
    (eo, el), d = check_full(wl.WORKLOADS["gqa_prefill_fp16"])
    assert d["grid"] > 0


def test_decode_hld_fp16_full():
    check_full(wl.WORKLOADS["decode_hld_fp16"])


def test_specdec_hld_fp16_full():
    check_full(wl.WORKLOADS["specdec_hld_fp16"])


def test_gqa_kvcache_bf16_reduced():
    w = wl.WORKLOADS["gqa_kvcache_bf16"]
    check_full(w, B=8, Lk=2048, seqlen_lo=1, seqlen_hi=2048)


def test_mla_specdec_bf16_reduced():
    w = wl.WORKLOADS["mla_specdec_bf16"]
    check_full(w, B=2, Hq=16, Hkv=16, Lk=2050)


@pytest.mark.parametrize("name,nrows", [("gqa_kvcache_bf16", 96), ("mla_specdec_bf16", 48),
                                        ("decode_hld_fp16", 32), ("specdec_hld_fp16", 64),
                                        ("mla_prefill2k_bf16", 48)])
def test_full_size_sampled_rows(name, nrows):
    """At the benchmark's full sizes and launch configuration, compare sampled rows."""
    w = wl.WORKLOADS[name]
    q, k, v, sl = wl.make_inputs(w, DEV)
    o, lse = run_workload(w, q, k, v, sl)
    rows = sample_rows(w.B, w.Hq, w.Lq, nrows, seed=7)
    og, lg = gather_rows(o, lse, rows)
    ro, rl = oracle_sampled(q, k, v, w.causal, rows, seqlens=sl)
    compare(og, lg, ro, rl, w.dtype, name)
    del q, k, v, o
    torch.cuda.empty_cache()


def test_kvcache_full_size_properties():
    """Properties that hold at any size: finite outputs and run-to-run bitwise
    determinism (the design has no atomics)."""
    w = wl.WORKLOADS["gqa_kvcache_bf16"]
    q, k, v, sl = wl.make_inputs(w, DEV)
    o1, l1 = run_workload(w, q, k, v, sl)
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = run_workload(w, q, k, v, sl)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.isfinite(o1).all() and torch.isfinite(l1).all()


# ------------------------------------------------------------------ shape sweep

SWEEP = []
_rng = np.random.default_rng(2024)
for kv in (1, 2, 63, 64, 65, 1023, 1025, 1500, 3000):
    for (dqk, dv) in ((64, 64), (128, 128), (192, 128)):
        qlen = int(_rng.choice([1, 2, 4, 8]))
        g = int(_rng.choice([1, 2, 4, 8]))
        dt = torch.float16 if _rng.random() < 0.5 else torch.bfloat16
        causal = bool(_rng.random() < 0.5)
        SWEEP.append((kv, qlen, g, dqk, dv, dt, causal))


@pytest.mark.parametrize("kv,qlen,g,dqk,dv,dt,causal", SWEEP,
                         ids=[f"kv{a}-q{b}-g{c}-d{d}_{e}-{str(f)[6:]}-c{int(h)}" for a, b, c, d, e, f, h in SWEEP])
def test_shape_sweep_fwd(kv, qlen, g, dqk, dv, dt, causal):
    w = wl.Workload("sweep", "fwd", "blhd", dt, B=2, Lq=qlen, Hq=2 * g, Hkv=2, Lk=kv, Dqk=dqk, Dv=dv,
                    causal=causal, seed=kv * 7 + qlen)
    check_full(w)


@pytest.mark.parametrize("g,qlen", [(1, 1), (2, 1), (4, 1), (8, 1), (4, 2), (8, 8), (1, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_kvcache_sweep(g, qlen, causal):
    w = wl.Workload("kvsweep", "kvcache", "blhd", torch.bfloat16, B=5, Lq=qlen, Hq=2 * g, Hkv=2,
                    Lk=1500, Dqk=128, Dv=128, causal=causal, seed=11 * g + qlen, seqlen_lo=0,
                    seqlen_hi=1500)
    check_full(w)


# ------------------------------------------------------------------ splits

@pytest.mark.parametrize("num_splits", [1, 2, 3, 7, 64, 1000])
def test_split_count_invariance(num_splits):
    w = wl.Workload("splits", "fwd", "blhd", torch.float16, B=2, Lq=4, Hq=8, Hkv=2, Lk=3000, Dqk=128,
                    Dv=128, causal=True, seed=77)
    (eo, el), d = check_full(w, num_splits=num_splits)
    if num_splits > 1:
        assert d["combine_launched"] == 1


def test_splits_agree_with_each_other():
    w = wl.Workload("splits", "fwd", "blhd", torch.bfloat16, B=1, Lq=1, Hq=4, Hkv=4, Lk=5000, Dqk=128,
                    Dv=128, causal=False, seed=78)
    q, k, v, _ = wl.make_inputs(w, DEV)
    outs = []
    for s in (1, 2, 5, 16):
        o, lse = run_workload(w, q, k, v, None, num_splits=s)
        outs.append((o.float().clone(), lse.clone()))
    for o, lse in outs[1:]:
        assert (o - outs[0][0]).abs().max().item() <= 1.6e-2
        assert ((lse - outs[0][1]).abs() / outs[0][1].abs().clamp(min=1)).max().item() <= 1e-5


# ------------------------------------------------------------------ edge cases

def test_kvcache_nan_poison_and_edge_lengths():
    """Slots beyond cache_seqlens hold NaN; lengths include 0, 1, 63, 64, 65, Lmax."""
    B, Lmax = 7, 200
    w = wl.Workload("poison", "kvcache", "blhd", torch.float16, B=B, Lq=2, Hq=8, Hkv=2, Lk=Lmax,
                    Dqk=128, Dv=128, causal=True, seed=5, seqlen_lo=0, seqlen_hi=Lmax)
    q, k, v, _ = wl.make_inputs(w, DEV)
    sl = torch.tensor([0, 1, 63, 64, 65, Lmax, 2], dtype=torch.int32)
    for b in range(B):
        k[b, int(sl[b]):] = float("nan")
        v[b, int(sl[b]):] = float("nan")
    o, lse = run_workload(w, q, k, v, sl)
    kc, vc = k.clone(), v.clone()
    for b in range(B):  # the oracle never reads past the length either; give it finite data
        kc[b, int(sl[b]):] = 0
        vc[b, int(sl[b]):] = 0
    ro, rl = oracle_full(q, kc, vc, True, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "poison")
    # b=0 has no key and b=1 (causal, Lq=2, one key) has an empty first row
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.all(torch.isneginf(lse[1][:, 0]))


def test_empty_rows_causal_lq_gt_lk():
    w = wl.Workload("empty", "fwd", "blhd", torch.float16, B=1, Lq=8, Hq=2, Hkv=1, Lk=3, Dqk=64, Dv=64,
                    causal=True, seed=9)
    check_full(w)


def test_zero_keys():
    w = wl.Workload("zero", "fwd", "blhd", torch.bfloat16, B=2, Lq=3, Hq=4, Hkv=2, Lk=0, Dqk=64, Dv=64,
                    causal=False, seed=10)
    q, k, v, _ = wl.make_inputs(w, DEV)
    o, lse = run_workload(w, q, k, v, None)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_overflow_shift_invariance():
    """Large common key offset (the pages' "ovf" robustness case): O is unchanged
    and lse moves by scale * q.u; checked against the oracle on the shifted keys."""
    w = wl.Workload("ovf", "fwd", "blhd", torch.float16, B=1, Lq=4, Hq=4, Hkv=4, Lk=777, Dqk=128,
                    Dv=128, causal=True, seed=12)
    q, k, v, _ = wl.make_inputs(w, DEV)
    k = (k.float() + 40.0).half()  # shifts every score by scale * 40 * sum(q): tens to ~100
    o, lse = run_workload(w, q, k, v, None)
    ro, rl = oracle_full(q, k, v, True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "ovf")


def test_output_canaries_and_strided_output():
    """Output written through a strided view inside a larger buffer: the bytes
    around it stay untouched."""
    w = wl.WORKLOADS["specdec_hld_fp16"]
    q, k, v, _ = wl.make_inputs(w, DEV, Lk=700)
    big = torch.full((w.Hq + 2, w.Lq, w.Dv + 64), 7.0, dtype=w.dtype, device=DEV)
    out = big[1:-1, :, 32:32 + w.Dv].unsqueeze(0).permute(0, 2, 1, 3)
    o, lse = fa.fa_fwd(q, k, v, causal=True, out=out)
    torch.cuda.synchronize()
    assert torch.all(big[0] == 7) and torch.all(big[-1] == 7)
    assert torch.all(big[:, :, :32] == 7) and torch.all(big[:, :, 32 + w.Dv:] == 7)
    ro, rl = oracle_full(q, k, v, True)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, "strided-out")


def test_determinism_bitwise():
    w = wl.WORKLOADS["specdec_hld_fp16"]
    q, k, v, _ = wl.make_inputs(w, DEV)
    o1, l1 = run_workload(w, q, k, v, None)
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = run_workload(w, q, k, v, None)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_no_lse_output():
    w = wl.WORKLOADS["decode_hld_fp16"]
    q, k, v, _ = wl.make_inputs(w, DEV, Lk=300)
    o, lse = fa.fa_fwd(q, k, v, return_lse=False)
    torch.cuda.synchronize()
    assert lse is None
    ro, rl = oracle_full(q, k, v, False)
    compare(o_to_numpy(o), None, ro, rl, w.dtype, "nolse")


# ------------------------------------------------------------------ errors

def test_errors_raise_without_launching():
    q = torch.zeros(1, 1, 4, 128, dtype=torch.float16, device=DEV)
    k = torch.zeros(1, 10, 2, 128, dtype=torch.float16, device=DEV)
    v = torch.zeros(1, 10, 2, 128, dtype=torch.bfloat16, device=DEV)
    n0 = fa.launch_count()
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(q, k, v)
    assert e.value.status == 1
    with pytest.raises(fa.FaError) as e:  # a V head dim above the largest kernel's 256
        fa.fa_fwd(q, k, torch.zeros(1, 10, 2, 264, dtype=torch.float16, device=DEV))
    assert e.value.status == 2
    ws_need = fa.fwd_workspace_size(q, k, k, num_splits=4)
    if ws_need:
        with pytest.raises((fa.FaError, ValueError)):
            fa.fa_fwd(q, k, k, num_splits=4, workspace=torch.empty(16, dtype=torch.uint8, device=DEV))
    assert fa.launch_count() == n0


# ------------------------------------------------------------------ both variants on one packed row

ONE_ROW = [(kv, d, dt) for kv in (1, 127, 129, 3000) for d in ((64, 64), (128, 128), (192, 128))
           for dt in (torch.float16, torch.bfloat16) if (kv + d[0] + (dt == torch.float16)) % 2 == 0 or kv == 3000]


@pytest.mark.parametrize("variant", ["mma", "scalar"])
@pytest.mark.parametrize("kv,d,dt", ONE_ROW, ids=[f"kv{a}-d{b[0]}_{b[1]}-{str(c)[6:]}" for a, b, c in ONE_ROW])
def test_one_row_both_variants(variant, kv, d, dt):
    """g * Lq == 1: the fp32 FMA variant and the tensor-core variant must both
    match the oracle (the library picks one of them by itself)."""
    fa.force_variant(fa.VARIANT_MMA if variant == "mma" else fa.VARIANT_SCALAR)
    w = wl.Workload("onerow", "fwd", "blhd", dt, B=3, Lq=1, Hq=4, Hkv=4, Lk=kv, Dqk=d[0], Dv=d[1],
                    causal=bool(kv % 2), seed=500 + kv)
    _, disp = check_full(w)
    assert disp["variant"] == (fa.VARIANT_MMA if variant == "mma" else fa.VARIANT_SCALAR)


@pytest.mark.parametrize("variant", ["mma", "scalar"])
@pytest.mark.parametrize("num_splits", [0, 1, 3, 50])
def test_one_row_kvcache_poisoned_tails(variant, num_splits):
    """Cache slots past each length hold NaN; lengths include 0, 1 and tile edges."""
    fa.force_variant(fa.VARIANT_MMA if variant == "mma" else fa.VARIANT_SCALAR)
    w = wl.Workload("onerow_kv", "kvcache", "blhd", torch.bfloat16, B=6, Lq=1, Hq=3, Hkv=3, Lk=700,
                    Dqk=128, Dv=128, causal=False, seed=610)
    q, k, v, _ = wl.make_inputs(w, DEV)
    sl = torch.tensor([0, 1, 127, 128, 129, 700], dtype=torch.int32)
    for b in range(w.B):
        k[b, int(sl[b]):] = float("nan")
        v[b, int(sl[b]):] = float("nan")
    o, lse = run_workload(w, q, k, v, sl, num_splits=num_splits)
    ro, rl = oracle_full(q, k, v, False, seqlens=sl)
    compare(o_to_numpy(o), lse_to_numpy(lse), ro, rl, w.dtype, w.name)


def test_scalar_variant_refuses_packed_rows():
    fa.force_variant(fa.VARIANT_SCALAR)
    w = wl.Workload("rows2", "fwd", "blhd", torch.float16, B=1, Lq=2, Hq=2, Hkv=2, Lk=64, Dqk=128, Dv=128,
                    causal=False, seed=1)
    q, k, v, _ = wl.make_inputs(w, DEV)
    with pytest.raises(fa.FaError, match="one packed row"):
        fa.fa_fwd(q, k, v)
