"""GPU parity of fa_fwd_varlen (through the C ABI) against the oracle's packed
form: decode and small-Q mixes (query lengths 0-8 per sequence), ragged key
lengths including 0, GQA, causal, head dims, split counts, and equality with
the dense call when every sequence has the same lengths."""
import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
import oracle

from helpers import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _status():
    yield
    torch.cuda.synchronize()
    fa.check_status()


def _packed(lq, lk, Hq, Hkv, d, dt, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    q = torch.randn(int(cq[-1]), Hq, d[0], generator=g, device=DEV).to(dt)
    k = torch.randn(int(ck[-1]), Hkv, d[0], generator=g, device=DEV).to(dt)
    v = torch.randn(int(ck[-1]), Hkv, d[1], generator=g, device=DEV).to(dt)
    return q, k, v, cq, ck


def _check(lq, lk, Hq=8, Hkv=2, d=(128, 128), dt=torch.bfloat16, causal=False, seed=0, num_splits=0):
    q, k, v, cq, ck = _packed(lq, lk, Hq, Hkv, d, dt, seed)
    o, lse = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), max(lq), max(lk), causal=causal,
                              num_splits=num_splits)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_varlen(q.cpu(), k.cpu(), v.cpu(), cq.numpy(), ck.numpy(), causal=causal)
    # compare as [total_q, Hq, Dv] rows; lse [Hq, total_q] -> rows of the same order
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, dt, "varlen")
    return o, lse


RNG = np.random.default_rng(7)
MIXES = [
    ([1] * 6, [1, 50, 127, 128, 129, 3000]),                        # decode, ragged contexts
    ([1, 2, 4, 8, 3], [700, 9, 1500, 64, 300]),                     # speculative / MTP mix
    (list(RNG.integers(1, 9, 20)), list(RNG.integers(0, 2000, 20))),  # 20 sequences, some with no keys
    ([4, 0, 2], [100, 50, 0]),                                      # an empty query range, an empty key range
]


@pytest.mark.parametrize("mix", range(len(MIXES)))
@pytest.mark.parametrize("causal", [False, True])
def test_mixes(mix, causal):
    lq, lk = MIXES[mix]
    _check([int(x) for x in lq], [int(x) for x in lk], causal=causal, seed=mix)


@pytest.mark.parametrize("d", [(64, 64), (192, 128), (256, 256)])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_head_dims(d, dt):
    _check([1, 3, 2], [400, 129, 1000], Hq=4, Hkv=4, d=d, dt=dt, causal=True, seed=d[0])


@pytest.mark.parametrize("g", [1, 4, 8, 16])
@pytest.mark.parametrize("num_splits", [0, 1, 5])
def test_gqa_and_splits(g, num_splits):
    _check([2, 1, 5], [300, 1025, 77], Hq=2 * g, Hkv=2, causal=True, seed=g, num_splits=num_splits)


def test_equal_lengths_match_dense_call():
    B, Lq, Lk, Hq, Hkv = 3, 2, 900, 8, 2
    q, k, v, cq, ck = _packed([Lq] * B, [Lk] * B, Hq, Hkv, (128, 128), torch.float16, 5)
    # one CTA per (sequence, kv head) in both calls: the same arithmetic, bit for bit
    o, lse = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), Lq, Lk, causal=True, num_splits=1)
    od, ld = fa.fa_fwd(q.view(B, Lq, Hq, 128), k.view(B, Lk, Hkv, 128), v.view(B, Lk, Hkv, 128), causal=True,
                       num_splits=1)
    torch.cuda.synchronize()
    assert torch.equal(o.view(B, Lq, Hq, 128), od)
    assert torch.equal(lse.view(Hq, B, Lq).permute(1, 0, 2), ld)


def test_flash_attn_varlen_func_wrapper():
    q, k, v, cq, ck = _packed([1, 2], [10, 20], 4, 4, (64, 64), torch.float16, 9)
    o = fa.flash_attn_varlen_func(q, k, v, cq.to(DEV), ck.to(DEV), 2, 20)
    o2, _ = fa.fa_fwd_varlen(q, k, v, cq.to(DEV), ck.to(DEV), 2, 20)
    torch.cuda.synchronize()
    assert o.shape == (3, 4, 64) and torch.equal(o, o2)
