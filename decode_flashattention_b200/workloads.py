"""Seeded synthetic workloads shaped like the pages' decode / small-Q cases.

This module only draws inputs (Q, K, V, cache lengths); it holds none of the
attention arithmetic, and both the CUDA path and the CPU oracle are fed from
it.  There is no dataset and no model weights: Q, K and V are i.i.d. N(0, 1)
drawn in fp32 with a seeded torch generator and rounded to the workload's
16-bit type; cache lengths are uniform integers.  Shapes follow the pages'
workloads (FlashAttention-style GQA forward from the MXFlashAttn README
example; the [numHeads, len, headDim] SmallQ interface and its validation
shapes -- Llama/Qwen 8B heads, kvLen 3000, qLen 1-8, MLA 192/128 -- from
"SmallQ FlashAttention for Ascend 910B"; the ~16K-token decode context of the
MXFlashAttn README's long-context regression).
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    call: str                 # "fwd" (dense K/V) or "kvcache" (per-batch cache lengths)
    layout: str               # "blhd": [B, L, H, D]; "hld": [H, L, D] storage (B = 1)
    dtype: torch.dtype
    B: int
    Lq: int
    Hq: int
    Hkv: int
    Lk: int                   # keys (fwd) or cache capacity Lmax (kvcache)
    Dqk: int
    Dv: int
    causal: bool
    seed: int
    seqlen_lo: int = 0        # kvcache: lengths uniform in [seqlen_lo, seqlen_hi]
    seqlen_hi: int = 0
    description: str = ""
    page: int = 0             # "paged": keys per cache block
    tensor_bound: bool = False  # prefill-shaped: measured against the tensor rate (flops), not HBM

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "gqa_prefill_fp16": Workload(
        "gqa_prefill_fp16", "fwd", "blhd", torch.float16, B=1, Lq=32, Hq=8, Hkv=2, Lk=128, Dqk=64,
        Dv=64, causal=True, seed=1001,
        description="flash_attn_func fwd fp16 B1 Lq32 Hq8 Hkv2 (GQA 4) Lk128 D64, causal"),
    "decode_hld_fp16": Workload(
        "decode_hld_fp16", "fwd", "hld", torch.float16, B=1, Lq=1, Hq=32, Hkv=32, Lk=4096, Dqk=128,
        Dv=128, causal=False, seed=1002,
        description="small-Q decode fp16 [H,L,D] H32 qLen1 D128 kvLen4096, non-causal"),
    "specdec_hld_fp16": Workload(
        "specdec_hld_fp16", "fwd", "hld", torch.float16, B=1, Lq=4, Hq=64, Hkv=64, Lk=3000, Dqk=128,
        Dv=128, causal=True, seed=1003,
        description="speculative small-Q fp16 [H,L,D] H64 qLen4 D128 kvLen3000, causal"),
    "gqa_kvcache_bf16": Workload(
        "gqa_kvcache_bf16", "kvcache", "blhd", torch.bfloat16, B=64, Lq=1, Hq=32, Hkv=8, Lk=16384,
        Dqk=128, Dv=128, causal=False, seed=1004, seqlen_lo=1, seqlen_hi=16384,
        description="batched GQA decode kvcache bf16 B64 Hq32 Hkv8 D128, seqlens U[1,16384]"),
    "mla_specdec_bf16": Workload(
        "mla_specdec_bf16", "fwd", "blhd", torch.bfloat16, B=8, Lq=8, Hq=128, Hkv=128, Lk=16384,
        Dqk=192, Dv=128, causal=True, seed=1005,
        description="MLA-shaped small-Q bf16 B8 qLen8 H128 Dqk192 Dv128 kvLen16384, causal"),
}

# Paged variants of the batched decode (not one of the five pages' shapes: the
# same GQA decode over a block-table cache, vLLM's usual 16-key pages and
# FlashAttention's 256-key pages).
for _pg in (16, 256):
    WORKLOADS[f"gqa_paged{_pg}_bf16"] = Workload(
        f"gqa_paged{_pg}_bf16", "paged", "blhd", torch.bfloat16, B=64, Lq=1, Hq=32, Hkv=8, Lk=16384,
        Dqk=128, Dv=128, causal=False, seed=1004, seqlen_lo=1, seqlen_hi=16384, page=_pg,
        description=f"batched GQA decode, paged cache ({_pg}-key blocks, shuffled) bf16 B64 Hq32 Hkv8 "
                    f"D128, seqlens U[1,16384]")

# GQA 8 with 4 speculative query positions over a batched KV cache: 32 packed
# rows per kv head, one unit of the tcgen05 split-KV kernel (GQA 2/4/8 in the
# MXFlashAttn README's capability table; qLen 1-8 in the SmallQ README).
WORKLOADS["gqa8_specdec_kvcache_bf16"] = Workload(
    "gqa8_specdec_kvcache_bf16", "kvcache", "blhd", torch.bfloat16, B=64, Lq=4, Hq=64, Hkv=8, Lk=16384, Dqk=128,
    Dv=128, causal=True, seed=1008, seqlen_lo=1, seqlen_hi=16384,
    description="batched GQA-8 speculative decode kvcache bf16 B64 qLen4 Hq64 Hkv8 D128, seqlens U[1,16384], causal")

# Head dim 256 (the SmallQ README's validation shapes include hd 256): GQA 4
# decode over an 8K context.
WORKLOADS["gqa_decode_hd256_bf16"] = Workload(
    "gqa_decode_hd256_bf16", "fwd", "blhd", torch.bfloat16, B=8, Lq=1, Hq=16, Hkv=4, Lk=8192, Dqk=256, Dv=256,
    causal=False, seed=1006, description="GQA decode bf16 B8 Hq16 Hkv4 D256 kvLen8192, non-causal")

# Long prefill (the tcgen05 kernel): GQA 4, 4K queries over 4K keys, causal.
WORKLOADS["gqa_prefill4k_bf16"] = Workload(
    "gqa_prefill4k_bf16", "fwd", "blhd", torch.bfloat16, B=1, Lq=4096, Hq=32, Hkv=8, Lk=4096, Dqk=128, Dv=128,
    causal=True, seed=1007, description="prefill bf16 B1 Lq4096 Hq32 Hkv8 D128 Lk4096, causal (tcgen05 kernel)",
    tensor_bound=True)

# Prefill-shaped call with the MLA head dims (192 / 128), GQA 4: the tcgen05
# split-KV kernel in row blocks of 64 (the dense tcgen05 kernel covers head
# dims 64 and 128 only).
WORKLOADS["mla_prefill2k_bf16"] = Workload(
    "mla_prefill2k_bf16", "fwd", "blhd", torch.bfloat16, B=1, Lq=2048, Hq=32, Hkv=8, Lk=8192, Dqk=192, Dv=128,
    causal=True, seed=1009, tensor_bound=True,
    description="prefill-shaped MLA head dims bf16 B1 Lq2048 Hq32 Hkv8 Dqk192 Dv128 Lk8192, causal "
                "(tcgen05 split-KV kernel, 64-row blocks)")

# The five configurations the metric is quoted on, in order (C1 ... C5).
CONFIG_IDS = {"C1": "gqa_prefill_fp16", "C2": "decode_hld_fp16", "C3": "specdec_hld_fp16",
              "C4": "gqa_kvcache_bf16", "C5": "mla_specdec_bf16"}
CONFIGS = list(CONFIG_IDS.values())

# the workload the bench reports by default: the largest single-GPU
# configuration (MLA-shaped speculative decode, 10.7 GB of K/V per call)
DEFAULT_BENCH = "mla_specdec_bf16"


def _randn(shape, gen, device, dtype, chunk_elems=1 << 28):
    """N(0,1) in fp32, rounded to dtype, generated in slices to bound the fp32 temp."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def draw_seqlens(w: Workload, seed: int | None = None) -> torch.Tensor:
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    return torch.randint(w.seqlen_lo, w.seqlen_hi + 1, (w.B,), generator=g, dtype=torch.int32)


def make_inputs(w: Workload, device="cuda", seed: int | None = None, **over):
    """Draw (q, k, v, seqlens) for workload w (fields may be overridden by keyword,
    e.g. Lk=256 for a reduced case).  q/k/v are 4-D [B, L, H, D] views; for the
    "hld" layout they are strided views of [H, L, D] storage.  seqlens is an
    int32 CPU tensor for kvcache workloads, else None."""
    if over:
        w = dataclasses.replace(w, **over)
    seed = w.seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    if w.layout == "hld":
        if w.B != 1 or w.Hq != w.Hkv:
            raise ValueError("the [H, L, D] layout has B = 1 and no GQA")
        qs = _randn((w.Hq, w.Lq, w.Dqk), gen, dev, w.dtype)
        ks = _randn((w.Hkv, w.Lk, w.Dqk), gen, dev, w.dtype)
        vs = _randn((w.Hkv, w.Lk, w.Dv), gen, dev, w.dtype)
        q, k, v = (t.unsqueeze(0).permute(0, 2, 1, 3) for t in (qs, ks, vs))
    else:
        q = _randn((w.B, w.Lq, w.Hq, w.Dqk), gen, dev, w.dtype)
        k = _randn((w.B, w.Lk, w.Hkv, w.Dqk), gen, dev, w.dtype)
        v = _randn((w.B, w.Lk, w.Hkv, w.Dv), gen, dev, w.dtype)
    if w.call == "paged":
        raise ValueError("paged workloads are drawn by make_paged_inputs")
    seqlens = draw_seqlens(w, seed) if w.call == "kvcache" else None
    return q, k, v, seqlens


def make_paged_inputs(w: Workload, device="cuda", seed: int | None = None, poison: bool = False, **over):
    """Draw (q, k_pages, v_pages, block_table, seqlens) for a paged workload.

    Each batch gets ceil(seqlens[b] / page) blocks from one pool of
    sum_b ceil(seqlens[b] / page) + 8 blocks, assigned in a seeded random
    order; table entries past a batch's blocks are -1.  K/V values are
    i.i.d. N(0, 1) like the dense workloads; with poison=True the pool's
    rows that no key addresses hold NaN.  block_table is an int32 device
    tensor [B, ceil(Lk / page)], seqlens an int32 CPU tensor."""
    if over:
        w = dataclasses.replace(w, **over)
    if w.page <= 0:
        raise ValueError("not a paged workload")
    seed = w.seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    sl = draw_seqlens(w, seed)
    mb = -(-w.Lk // w.page)
    used = [-(-int(n) // w.page) for n in sl]
    nb = sum(used) + 8
    order = torch.randperm(nb, generator=torch.Generator().manual_seed(seed + 1))
    table = torch.full((w.B, mb), -1, dtype=torch.int32)
    pos = 0
    for b in range(w.B):
        table[b, :used[b]] = order[pos:pos + used[b]].to(torch.int32)
        pos += used[b]
    q = _randn((w.B, w.Lq, w.Hq, w.Dqk), gen, dev, w.dtype)
    kp = _randn((nb, w.page, w.Hkv, w.Dqk), gen, dev, w.dtype)
    vp = _randn((nb, w.page, w.Hkv, w.Dv), gen, dev, w.dtype)
    if poison:
        live = torch.zeros(nb, w.page, dtype=torch.bool)
        for b in range(w.B):
            for j0 in range(0, int(sl[b]), w.page):
                live[int(table[b, j0 // w.page]), :min(w.page, int(sl[b]) - j0)] = True
        dead = (~live).to(dev)
        kp[dead] = float("nan")
        vp[dead] = float("nan")
    return q, kp, vp, table.to(dev), sl


def empty_output(w: Workload, q: torch.Tensor) -> torch.Tensor:
    """Output buffer in the workload's layout ([H, Lq, Dv] storage for "hld")."""
    if w.layout == "hld":
        return torch.empty((w.Hq, w.Lq, w.Dv), dtype=w.dtype, device=q.device).unsqueeze(0).permute(0, 2, 1, 3)
    return torch.empty((w.B, w.Lq, w.Hq, w.Dv), dtype=w.dtype, device=q.device)


def kv_bytes(w: Workload, seqlens=None) -> int:
    """Algorithmic K/V bytes of one call: every key row a batch attends to
    (cache_seqlens[b] rows, or Lk) is read once for K (Dqk) and once for V (Dv)."""
    elt = 2
    if w.call in ("kvcache", "paged"):
        total = int(torch.as_tensor(seqlens).to(torch.int64).sum())
    else:
        total = w.B * w.Lk
    return total * w.Hkv * (w.Dqk + w.Dv) * elt


def attn_flops(w: Workload, seqlens=None) -> int:
    """Multiply-add flops of one call, 2 * (Dqk + Dv) per visible (row, key)
    pair: every query row of every head against the keys it sees (all n
    keys, or j <= i + n - Lq under the bottom-right causal mask)."""
    if w.call in ("kvcache", "paged"):
        ns = [int(x) for x in torch.as_tensor(seqlens).tolist()]
    else:
        ns = [w.Lk] * w.B
    vis = 0
    for n in ns:
        if w.causal:
            vis += sum(max(0, min(n, i + n - w.Lq + 1)) for i in range(w.Lq))
        else:
            vis += n * w.Lq
    return 2 * (w.Dqk + w.Dv) * vis * w.Hq


def tokens_per_call(w: Workload) -> int:
    return w.B * w.Lq
