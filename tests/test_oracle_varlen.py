"""Pins of the oracle's packed variable-length form (CPU only): each packed
sequence equals the dense definition on its own slice (checked against
torch fp64 SDPA, a library routine), sequences do not see each other, and
an empty key range gives O = 0, lse = -inf."""
import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa(q, k, v, causal):
    # q [Lq, Hq, D], k/v [n, Hkv, D] in fp64: repeat kv heads, explicit bottom-right mask
    Lq, Hq, D = q.shape
    n, Hkv = k.shape[0], k.shape[1]
    g = Hq // Hkv
    kk = k.repeat_interleave(g, dim=1).permute(1, 0, 2)
    vv = v.repeat_interleave(g, dim=1).permute(1, 0, 2)
    qq = q.permute(1, 0, 2)
    s = qq @ kk.transpose(1, 2) / math.sqrt(D)
    if causal:
        i = torch.arange(Lq)[:, None]
        j = torch.arange(n)[None, :]
        s = s.masked_fill(j > i + n - Lq, -math.inf)
    lse = torch.logsumexp(s, -1)
    o = torch.softmax(s, -1) @ vv
    return o.permute(1, 0, 2), lse


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_definition(causal):
    rng = np.random.default_rng(1)
    lq = [1, 3, 8, 2]
    lk = [5, 9, 20, 2]
    cq = np.concatenate([[0], np.cumsum(lq)])
    ck = np.concatenate([[0], np.cumsum(lk)])
    Hq, Hkv, D = 4, 2, 8
    q = torch.from_numpy(rng.standard_normal((cq[-1], Hq, D)))
    k = torch.from_numpy(rng.standard_normal((ck[-1], Hkv, D)))
    v = torch.from_numpy(rng.standard_normal((ck[-1], Hkv, D)))
    o, lse = oracle.attention_varlen(q, k, v, cq, ck, causal=causal)
    for b in range(len(lq)):
        ro, rl = _sdpa(q[cq[b]:cq[b + 1]], k[ck[b]:ck[b + 1]], v[ck[b]:ck[b + 1]], causal)
        assert np.allclose(o[cq[b]:cq[b + 1]], ro.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[:, cq[b]:cq[b + 1]], rl.numpy(), rtol=0, atol=1e-12)


def test_sequences_are_isolated_and_empty_keys_give_zero():
    rng = np.random.default_rng(2)
    cq, ck = np.array([0, 2, 4]), np.array([0, 0, 6])
    q = torch.from_numpy(rng.standard_normal((4, 2, 4)))
    k = torch.from_numpy(rng.standard_normal((6, 2, 4)))
    v = torch.from_numpy(rng.standard_normal((6, 2, 4)))
    o, lse = oracle.attention_varlen(q, k, v, cq, ck)
    assert np.all(o[:2] == 0) and np.all(np.isneginf(lse[:, :2]))
    # changing sequence 1's keys leaves sequence 0 alone and vice versa
    k2 = k.clone()
    k2[3] += 5.0
    o2, _ = oracle.attention_varlen(q, k2, v, cq, ck)
    assert np.array_equal(o2[:2], o[:2]) and not np.array_equal(o2[2:], o[2:])
