"""Pins of the oracle's paged-cache addressing (CPU only).

Key j of batch b lives at row j % page of block block_table[b, j // page]
(the block-table convention of FlashAttention's flash_attn_with_kvcache,
which the MXFlashAttn README's kvcache interface follows; its capability
table lists paged KV caches).  The pins: a zero query averages exactly the
V rows the table addresses (a closed form that fixes the page / row
arithmetic), a paged cache equals the dense cache it was cut from under any
block permutation, and planted addressing mistakes are caught.
"""
import numpy as np
import pytest
import torch

import oracle


def _paged_from_dense(dense, page, rng, extra_blocks=3):
    """Cut a dense [B, L, H, D] cache into shuffled pages; returns (pages, table)."""
    B, L, H, D = dense.shape
    mb = -(-L // page)
    nb = B * mb + extra_blocks
    perm = rng.permutation(nb)
    pages = torch.randn(nb, page, H, D, dtype=torch.float64).to(dense.dtype)  # unused blocks: noise
    table = np.zeros((B, mb), dtype=np.int64)
    for b in range(B):
        for i in range(mb):
            blk = int(perm[b * mb + i])
            table[b, i] = blk
            rows = dense[b, i * page:(i + 1) * page]
            pages[blk, :rows.shape[0]] = rows
    return pages, table


def test_zero_query_averages_the_addressed_rows():
    # page 2; batch 0 -> blocks [3, 1, 0], 5 keys; batch 1 -> blocks [2, 0], 3 keys
    nb, page, H, D = 4, 2, 1, 3
    v = torch.arange(nb * page * H * D, dtype=torch.float64).reshape(nb, page, H, D)
    k = torch.randn(nb, page, H, D, dtype=torch.float64)
    table = np.array([[3, 1, 0], [2, 0, 0]])
    sl = np.array([5, 3])
    q = torch.zeros(2, 1, 1, D, dtype=torch.float64)
    o, lse = oracle.attention_paged(q, k, v, table, sl)
    want0 = (v[3, 0, 0] + v[3, 1, 0] + v[1, 0, 0] + v[1, 1, 0] + v[0, 0, 0]) / 5
    want1 = (v[2, 0, 0] + v[2, 1, 0] + v[0, 0, 0]) / 3
    assert np.allclose(o[0, 0, 0], want0.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(o[1, 0, 0], want1.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(lse[:, 0, 0], np.log([5, 3]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("page", [1, 2, 4, 16])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_paged_equals_dense_under_any_block_order(page, dt):
    rng = np.random.default_rng(page)
    B, L, Hq, Hkv, D, Lq = 3, 37, 4, 2, 8, 2
    q = torch.randn(B, Lq, Hq, D, dtype=torch.float64).to(dt)
    kd = torch.randn(B, L, Hkv, D, dtype=torch.float64).to(dt)
    vd = torch.randn(B, L, Hkv, D, dtype=torch.float64).to(dt)
    sl = np.array([0, 17, 37])
    kp, table = _paged_from_dense(kd, page, rng)
    vp_, table2 = _paged_from_dense(vd, page, np.random.default_rng(page))  # same permutation
    assert np.array_equal(table, table2)
    for causal in (False, True):
        o1, l1 = oracle.attention_paged(q, kp, vp_, table, sl, causal=causal)
        o2, l2 = oracle.attention(q, kd, vd, causal=causal, seqlens=sl)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_entries_past_the_length_are_never_read():
    nb, page, H, D = 3, 4, 1, 2
    k = torch.randn(nb, page, H, D, dtype=torch.float64)
    v = torch.randn(nb, page, H, D, dtype=torch.float64)
    q = torch.randn(1, 1, 1, D, dtype=torch.float64)
    a = oracle.attention_paged(q, k, v, np.array([[1, 2, 0]]), [5])
    b = oracle.attention_paged(q, k, v, np.array([[1, 2, 7]]), [5])  # 7: no such block, never needed
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    with pytest.raises(ValueError):
        oracle.attention_paged(q, k, v, np.array([[1, 7, 0]]), [5])  # needed, out of range


def _mutant_gather(kind):
    def g(pages, table, seqlens):
        nb, page, H, D = pages.shape
        B, mb = table.shape
        out = torch.zeros((B, mb * page, H, D), dtype=pages.dtype)
        for b in range(B):
            for j in range(int(seqlens[b])):
                if kind == "row_page_swapped":
                    blk, row = table[b, j % mb], (j // mb) % page
                elif kind == "table_transposed":
                    blk, row = table.T.reshape(B, mb)[b, j // page], j % page
                else:  # "block_off_by_one"
                    blk, row = table[b, j // page], (j + 1) % page
                out[b, j] = pages[int(blk), int(row)]
        return out
    return g


@pytest.mark.parametrize("kind", ["row_page_swapped", "table_transposed", "block_off_by_one"])
def test_pins_catch_planted_addressing_mistake(kind, monkeypatch):
    monkeypatch.setattr(oracle, "gather_pages", _mutant_gather(kind))
    caught = False
    try:
        test_zero_query_averages_the_addressed_rows()
    except AssertionError:
        caught = True
    if not caught:
        try:
            test_paged_equals_dense_under_any_block_order(2, torch.float16)
        except AssertionError:
            caught = True
    assert caught, kind
