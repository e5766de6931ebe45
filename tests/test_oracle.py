"""Pins for the fp64 oracle (CPU only).

The oracle is trusted only after it agrees with things other than itself:
exhaustive format decoding against numpy / torch, hand-worked closed forms
(tests/golden/closed_forms.json), torch's fp64 scaled_dot_product_attention
(a library routine), invariants of the definition, and the pages' tiled
online-softmax algorithm.  The last test shows that each plausible mistake
(dropped scale, wrong causal corner, wrong GQA map, swapped operands, wrong
log base, off-by-one length) fails at least one of these pins.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import online

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- formats

def test_f16_decode_exhaustive(oracle_mod):
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_bits_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decode_exhaustive(oracle_mod):
    bits = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_bits_to_f64(int(b) & 0xFFFF) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- helpers

def rand(rng, *shape):
    return rng.standard_normal(shape)


def oracle_attn(q, k, v, causal=False, scale=None, seqlens=None):
    return oracle.attention(np.asarray(q, np.float64), np.asarray(k, np.float64),
                            np.asarray(v, np.float64), causal=causal, scale=scale,
                            seqlens=seqlens, nthreads=2)


# ---------------------------------------------------------------- closed forms

def load_golden():
    with open(os.path.join(GOLDEN, "closed_forms.json")) as f:
        return json.load(f)


def pin_golden(attn):
    g = load_golden()
    fails = []
    c = g["two_key_softmax"]
    o, lse = attn(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]), causal=False,
                  scale=c["scale"])
    if not (np.allclose(o, c["o"], rtol=0, atol=1e-14) and np.allclose(lse, c["lse"], atol=1e-14)):
        fails.append("two_key_softmax")
    c = g["zero_query_bottom_right_causal"]
    Lq, vv = c["Lq"], np.array(c["v"])
    n = vv.shape[0]
    q = np.zeros((1, Lq, 1, 4))
    k = rand(np.random.default_rng(5), 1, n, 1, 4)
    v = vv.reshape(1, n, 1, 1)
    o, lse = attn(q, k, v, causal=True)
    if not (np.allclose(o[0, :, 0, 0], c["o"], atol=1e-14) and np.allclose(lse[0, 0], c["lse"], atol=1e-14)):
        fails.append("zero_query_bottom_right_causal")
    c = g["zero_query_cache_seqlens"]
    sl = np.array(c["seqlens"], dtype=np.int32)
    vv = np.array(c["v"])
    n = vv.shape[0]
    B = sl.shape[0]
    q = np.zeros((B, 1, 1, 4))
    k = rand(np.random.default_rng(6), B, n, 1, 4)
    v = np.broadcast_to(vv.reshape(1, n, 1, 1), (B, n, 1, 1)).copy()
    o, lse = attn(q, k, v, causal=False, seqlens=sl)
    want_lse = np.array([float(x) for x in c["lse"]])
    ok = np.allclose(o[:, 0, 0, 0], c["o"], atol=1e-14)
    ok &= np.array_equal(np.isinf(lse[:, 0, 0]), np.isinf(want_lse))
    fin = ~np.isinf(want_lse)
    ok &= np.allclose(lse[fin, 0, 0], want_lse[fin], atol=1e-14)
    if not ok:
        fails.append("zero_query_cache_seqlens")
    return fails


def pin_kvlen1(attn):
    rng = np.random.default_rng(11)
    q, k, v = rand(rng, 2, 3, 4, 16), rand(rng, 2, 1, 2, 16), rand(rng, 2, 1, 2, 8)
    o, lse = attn(q, k, v, causal=False)
    fails = []
    for b in range(2):
        for hq in range(4):
            hkv = hq // 2
            for i in range(3):
                if not np.allclose(o[b, i, hq], v[b, 0, hkv], atol=1e-13):
                    fails.append("kvlen1_o")
                s = float(q[b, i, hq] @ k[b, 0, hkv]) / 4.0  # scale 1/sqrt(16)
                if abs(lse[b, hq, i] - s) > 1e-12:
                    fails.append("kvlen1_lse")
    return sorted(set(fails))


def pin_identical_keys(attn):
    rng = np.random.default_rng(12)
    Lq, n, D = 4, 9, 8
    q = rand(rng, 1, Lq, 2, D)
    key = rand(rng, D)
    k = np.broadcast_to(key, (1, n, 1, D)).copy()
    v = rand(rng, 1, n, 1, 5)
    o, lse = attn(q, k, v, causal=True)
    fails = []
    for h in range(2):
        for i in range(Lq):
            cnt = i + n - Lq + 1
            if not np.allclose(o[0, i, h], v[0, :cnt, 0].mean(axis=0), atol=1e-13):
                fails.append("identical_keys_o")
            want = float(q[0, i, h] @ key) / math.sqrt(D) + math.log(cnt)
            if abs(lse[0, h, i] - want) > 1e-12:
                fails.append("identical_keys_lse")
    return sorted(set(fails))


def pin_zero_query(attn):
    """Q = 0: O_i = mean of visible V rows, lse_i = ln |J_i| (pins the causal
    corner and the cache_seqlens bound exactly)."""
    rng = np.random.default_rng(13)
    B, Lq, Lk, D = 3, 5, 12, 4
    sl = np.array([12, 7, 3], dtype=np.int32)
    q = np.zeros((B, Lq, 2, D))
    k = rand(rng, B, Lk, 1, D)
    v = rand(rng, B, Lk, 1, 6)
    fails = []
    for causal in (False, True):
        o, lse = attn(q, k, v, causal=causal, seqlens=sl)
        for b in range(B):
            n = int(sl[b])
            for i in range(Lq):
                cnt = min(n, i + n - Lq + 1) if causal else n
                for h in range(2):
                    if cnt <= 0:
                        if not (np.all(o[b, i, h] == 0) and lse[b, h, i] == -math.inf):
                            fails.append("zero_query_empty_row")
                        continue
                    if not np.allclose(o[b, i, h], v[b, :cnt, 0].mean(axis=0), atol=1e-13):
                        fails.append(f"zero_query_o_causal{int(causal)}")
                    if abs(lse[b, h, i] - math.log(cnt)) > 1e-12:
                        fails.append(f"zero_query_lse_causal{int(causal)}")
    return sorted(set(fails))


# ---------------------------------------------------------------- library routine

def torch_reference(q, k, v, causal, scale, seqlens):
    """torch fp64 SDPA with an explicit visibility mask and K/V heads repeated
    to the query heads; lse from torch.logsumexp of the masked scaled scores."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)  # [B, Hq, Lq, D]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    B, Hq, Lq, _ = qt.shape
    Lk = kt.shape[2]
    g = Hq // kt.shape[1]
    kt = kt.repeat_interleave(g, dim=1)
    vt = vt.repeat_interleave(g, dim=1)
    i = torch.arange(Lq).view(Lq, 1)
    j = torch.arange(Lk).view(1, Lk)
    masks = []
    for b in range(B):
        n = int(seqlens[b]) if seqlens is not None else Lk
        m = (j < n).expand(Lq, Lk)
        if causal:
            m = m & (j <= i + n - Lq)
        masks.append(m)
    mask = torch.stack(masks).view(B, 1, Lq, Lk)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    s = (qt @ kt.transpose(-1, -2)) * scale
    lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def pin_torch_sdpa(attn, cases=12):
    rng = np.random.default_rng(14)
    fails = []
    for c in range(cases):
        B = int(rng.integers(1, 3))
        Lq = int(rng.integers(1, 9))
        Lk = int(rng.integers(Lq, 40))
        Hkv = int(rng.integers(1, 3))
        g = int(rng.choice([1, 2, 4]))
        D = int(rng.choice([8, 16]))
        Dv = int(rng.choice([8, 12]))
        causal = bool(c % 2)
        sl = rng.integers(Lq, Lk + 1, size=B).astype(np.int32) if c % 3 == 0 else None
        q, k, v = rand(rng, B, Lq, Hkv * g, D), rand(rng, B, Lk, Hkv, D), rand(rng, B, Lk, Hkv, Dv)
        scale = 1.0 / math.sqrt(D)
        o, lse = attn(q, k, v, causal=causal, seqlens=sl)
        ro, rl = torch_reference(q, k, v, causal, scale, sl)
        if not np.allclose(o, ro, atol=1e-12, rtol=0):
            fails.append("sdpa_o")
        if not np.allclose(lse, rl, atol=1e-12, rtol=0):
            fails.append("sdpa_lse")
    return sorted(set(fails))


# ---------------------------------------------------------------- invariants

def pin_invariants(attn):
    rng = np.random.default_rng(15)
    fails = []
    B, Lq, Hkv, g, Lk, D, Dv = 2, 3, 2, 2, 17, 8, 6
    q, k, v = rand(rng, B, Lq, Hkv * g, D), rand(rng, B, Lk, Hkv, D), rand(rng, B, Lk, Hkv, Dv)
    o, lse = attn(q, k, v, causal=False)
    # KV permutation (non-causal)
    perm = rng.permutation(Lk)
    o2, lse2 = attn(q, k[:, perm], v[:, perm], causal=False)
    if not (np.allclose(o, o2, atol=1e-13) and np.allclose(lse, lse2, atol=1e-12)):
        fails.append("permutation")
    # shift of every key by the same vector u (large: the overflow case)
    u = 40.0 * rand(rng, D)
    o3, lse3 = attn(q, k + u, v, causal=False)
    shift = np.einsum("bihd,d->bhi", q, u) / math.sqrt(D)
    if not (np.allclose(o, o3, atol=1e-9) and np.allclose(lse3 - lse, shift, atol=1e-8)):
        fails.append("shift")
    # GQA equals an explicit repeat of the kv heads
    o4, lse4 = attn(q, np.repeat(k, g, axis=2), np.repeat(v, g, axis=2), causal=False)
    if not (np.allclose(o, o4, atol=1e-13) and np.allclose(lse, lse4, atol=1e-12)):
        fails.append("gqa_repeat")
    # causal with one query row equals non-causal
    o5, lse5 = attn(q[:, :1], k, v, causal=True)
    o6, lse6 = attn(q[:, :1], k, v, causal=False)
    if not (np.allclose(o5, o6, atol=1e-14) and np.allclose(lse5, lse6, atol=1e-14)):
        fails.append("causal_lq1")
    # cache_seqlens = n equals a slice of the first n keys
    sl = np.array([11, 4], dtype=np.int32)
    o7, lse7 = attn(q, k, v, causal=True, seqlens=sl)
    for b in range(B):
        n = int(sl[b])
        o8, lse8 = attn(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], causal=True)
        if not (np.allclose(o7[b:b + 1], o8, atol=1e-14) and np.allclose(lse7[b:b + 1], lse8, atol=1e-14)):
            fails.append("seqlens_slice")
    # convex hull: every output lies within the visible value rows' range
    for b in range(B):
        n = int(sl[b])
        for h in range(Hkv * g):
            for i in range(Lq):
                cnt = min(n, i + n - Lq + 1)
                vv = v[b, :cnt, h // g]
                if np.any(o7[b, i, h] < vv.min(axis=0) - 1e-12) or np.any(o7[b, i, h] > vv.max(axis=0) + 1e-12):
                    fails.append("convex_hull")
    return sorted(set(fails))


ALL_PINS = [pin_golden, pin_kvlen1, pin_identical_keys, pin_zero_query, pin_torch_sdpa,
            pin_invariants]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_passes_pin(oracle_mod, pin):
    assert pin(oracle_attn) == []


# ---------------------------------------------------------------- 16-bit inputs

@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_16bit_inputs_equal_f64_of_decoded_values(oracle_mod, dt):
    g = torch.Generator().manual_seed(21)
    q = torch.randn(2, 4, 8, 64, generator=g).to(dt)
    k = torch.randn(2, 37, 2, 64, generator=g).to(dt)
    v = torch.randn(2, 37, 2, 64, generator=g).to(dt)
    sl = np.array([37, 20], dtype=np.int32)
    o, lse = oracle.attention(q, k, v, causal=True, seqlens=sl, nthreads=3)
    o2, lse2 = oracle_attn(q.double().numpy(), k.double().numpy(), v.double().numpy(), True,
                           None, sl)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_strided_hld_layout(oracle_mod):
    """[H, L, D] storage viewed as [1, L, H, D] through strides."""
    g = torch.Generator().manual_seed(22)
    H, Lq, Lk, D = 4, 2, 29, 32
    qs = torch.randn(H, Lq, D, generator=g).half()
    ks = torch.randn(H, Lk, D, generator=g).half()
    vs = torch.randn(H, Lk, D, generator=g).half()
    q, k, v = (t.unsqueeze(0).permute(0, 2, 1, 3) for t in (qs, ks, vs))
    assert not q.is_contiguous()
    o, lse = oracle.attention(q, k, v, causal=True)
    o2, lse2 = oracle.attention(q.contiguous(), k.contiguous(), v.contiguous(), causal=True)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(23)
    q, k, v = rand(rng, 2, 3, 4, 8), rand(rng, 2, 10, 2, 8), rand(rng, 2, 10, 2, 8)
    o, lse = oracle_attn(q, k, v, causal=True)
    rows = np.array([[1, 3, 2], [0, 0, 0], [1, 1, 1]])
    o2, lse2 = oracle.attention(q, k, v, causal=True, rows=rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(o2[r], o[b, i, h]) and lse2[r] == lse[b, h, i]


def test_invalid_arguments_rejected(oracle_mod):
    q, k, v = np.zeros((1, 1, 3, 4)), np.zeros((1, 2, 2, 4)), np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):
        oracle.attention(q, k, v)  # Hq % Hkv != 0
    q = np.zeros((1, 1, 2, 4))
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, seqlens=[3])  # seqlen > Lk


# ---------------------------------------------------------------- the tiled algorithm

def test_online_equals_definition_any_tile_and_split(oracle_mod):
    rng = np.random.default_rng(31)
    for trial in range(6):
        B, Lq, Hkv, g = 2, int(rng.integers(1, 6)), 2, int(rng.choice([1, 2, 4]))
        Lk, D, Dv = int(rng.integers(5, 70)), 16, 8
        q, k, v = rand(rng, B, Lq, Hkv * g, D), rand(rng, B, Lk, Hkv, D), rand(rng, B, Lk, Hkv, Dv)
        sl = rng.integers(0, Lk + 1, size=B).astype(np.int32)
        causal = bool(trial % 2)
        tile = int(rng.integers(1, 20))
        nsplit = int(rng.integers(1, 6))

        def bounds(b, n, nsplit=nsplit):
            cuts = sorted(set(int(x) for x in rng.integers(1, max(n, 2), size=nsplit - 1)))
            return [0] + [c for c in cuts if 0 < c < n]

        o, lse = oracle_attn(q, k, v, causal=causal, seqlens=sl)
        o2, lse2 = online.attention_online(q, k, v, causal=causal, seqlens=sl, tile=tile,
                                           split_bounds=bounds)
        assert np.allclose(o, o2, atol=1e-12)
        assert np.array_equal(np.isinf(lse), np.isinf(lse2))
        fin = ~np.isinf(lse)
        assert np.allclose(lse[fin], lse2[fin], atol=1e-12)


def test_combine_of_single_split_is_identity():
    o = np.array([0.5, -2.0])
    oo, L = online.combine([o], [3.25])
    assert np.array_equal(oo, o) and L == 3.25
    oo, L = online.combine([o, o], [-math.inf, -math.inf])
    assert np.all(oo == 0) and L == -math.inf


def test_online_pins(oracle_mod):
    """The online algorithm passes the same pins as the definition."""
    def attn(q, k, v, causal=False, scale=None, seqlens=None):
        return online.attention_online(q, k, v, causal=causal, scale=scale, seqlens=seqlens,
                                       tile=3, split_bounds=lambda b, n: [0] + ([n // 2] if n > 1 else []))
    for pin in ALL_PINS:
        assert pin(attn) == [], pin.__name__


# ---------------------------------------------------------------- the pins catch mistakes

def _mutant(kind):
    """A definition with one plausible mistake planted (CPU, test-only)."""
    def attn(q, k, v, causal=False, scale=None, seqlens=None):
        q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
        B, Lq, Hq, D = q.shape
        _, Lk, Hkv, _ = k.shape
        g = Hq // Hkv
        if scale is None:
            scale = 1.0 / math.sqrt(D)
        if kind == "no_scale":
            scale = 1.0
        o = np.zeros((B, Lq, Hq, v.shape[3]))
        lse = np.full((B, Hq, Lq), -math.inf)
        for b in range(B):
            n = int(seqlens[b]) if seqlens is not None else Lk
            if kind == "seqlen_off_by_one" and seqlens is not None:
                n = max(0, n - 1)
            for h in range(Hq):
                hk = h % Hkv if kind == "gqa_modulo" else h // g
                for i in range(Lq):
                    last = n - 1
                    if causal:
                        last = min(last, i if kind == "top_left_causal" else i + n - Lq)
                    if last < 0:
                        continue
                    kk, vv = k[b, :last + 1, hk], v[b, :last + 1, hk]
                    if kind == "swap_kv" and kk.shape[1] == vv.shape[1]:
                        kk, vv = vv, kk
                    s = scale * (kk @ q[b, i, h])
                    m = s.max()
                    p = np.exp(s - m)
                    o[b, i, h] = p @ vv / p.sum()
                    lse[b, h, i] = (m + math.log(p.sum())) / (math.log(2) if kind == "log2_lse" else 1.0)
        return o, lse
    return attn


@pytest.mark.parametrize("kind", ["no_scale", "top_left_causal", "gqa_modulo", "swap_kv",
                                  "log2_lse", "seqlen_off_by_one"])
def test_pins_catch_planted_mistake(kind):
    failed = []
    for pin in ALL_PINS:
        failed += pin(_mutant(kind))
    assert failed, f"no pin caught the planted mistake {kind}"


def test_correct_numpy_definition_passes_pins():
    assert sum((pin(_mutant("none")) for pin in ALL_PINS), []) == []
