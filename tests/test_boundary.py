"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/fa.h declares, rejects malformed calls on the host before
touching a device, and its host-side work partition has the properties the
kernels rely on."""
import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

import decode_flashattention_b200 as fa
from decode_flashattention_b200 import FaTensor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA, TIMEOUT = range(6)


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = fa.load_library()
    names = header_functions()
    assert "fa_fwd" in names and "fa_decode_kvcache" in names
    for n in names:
        assert hasattr(lib, n), n


def test_version_string():
    assert b"sm_100a" in fa.load_library().fa_version()


def desc(shape, dtype=0, stride=None, ptr=0x10000):
    d = FaTensor()
    d.data = ptr
    d.dtype = dtype
    if stride is None:
        stride = [int(np.prod(shape[i + 1:])) for i in range(4)]
    for i in range(4):
        d.shape[i] = shape[i]
        d.stride[i] = stride[i]
    return d


def call_fwd(q, k, v, o, causal=0, scale=0.0, lse=None):
    lib = fa.load_library()
    return lib.fa_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(o) if o else None,
                      lse, causal, scale, 0, None, 0, None)


GOOD = dict(q=[1, 1, 8, 128], k=[1, 64, 2, 128], v=[1, 64, 2, 128], o=[1, 1, 8, 128])


def good(name, **kw):
    return desc(GOOD[name], **kw)


@pytest.mark.parametrize("case,expect", [
    ("dtype_mismatch", INVALID), ("bad_gqa", INVALID), ("head_dim_264", UNSUPPORTED), ("head_dim_12", UNSUPPORTED),
    ("head_dim_v_264", UNSUPPORTED),
    ("last_dim_strided", UNSUPPORTED), ("stride_not_16B", UNSUPPORTED), ("misaligned", UNSUPPORTED),
    ("null_o", INVALID), ("batch_mismatch", INVALID), ("nan_scale", INVALID), ("fp32", UNSUPPORTED),
    ("too_many_row_blocks", UNSUPPORTED), ("null_data", INVALID), ("o_shape", INVALID),
])
def test_host_validation(case, expect):
    q, k, v, o = good("q"), good("k"), good("v"), good("o")
    scale = 0.0
    if case == "dtype_mismatch":
        v = good("v", dtype=1)
    elif case == "bad_gqa":
        q = desc([1, 1, 3, 128]); o = desc([1, 1, 3, 128])
    elif case == "head_dim_264":  # above the largest kernel's 256
        q, k, v, o = desc([1, 1, 8, 264]), desc([1, 64, 2, 264]), desc([1, 64, 2, 264]), desc([1, 1, 8, 264])
    elif case == "head_dim_12":  # rows of 24 bytes: no 16-byte row stride
        q, k, v, o = desc([1, 1, 8, 12]), desc([1, 64, 2, 12]), desc([1, 64, 2, 12]), desc([1, 1, 8, 12])
    elif case == "head_dim_v_264":
        v, o = desc([1, 64, 2, 264]), desc([1, 1, 8, 264])
    elif case == "last_dim_strided":
        k = desc([1, 64, 2, 128], stride=[64 * 2 * 256, 2 * 256, 256, 2])
    elif case == "stride_not_16B":
        k = desc([1, 64, 2, 128], stride=[64 * 2 * 132, 2 * 132, 132, 1])
    elif case == "misaligned":
        k = good("k", ptr=0x10008)
    elif case == "null_o":
        o = None
    elif case == "batch_mismatch":
        k = desc([2, 64, 2, 128])
    elif case == "nan_scale":
        scale = float("nan")
    elif case == "fp32":
        q, k, v, o = good("q", dtype=2), good("k", dtype=2), good("v", dtype=2), good("o", dtype=2)
    elif case == "too_many_row_blocks":
        q, o = desc([9000, 1, 8, 128]), desc([9000, 1, 8, 128])
        k, v = desc([9000, 64, 2, 128]), desc([9000, 64, 2, 128])
    elif case == "null_data":
        q = good("q", ptr=0)
    elif case == "o_shape":
        o = desc([1, 2, 8, 128])
    assert call_fwd(q, k, v, o, scale=scale) == expect
    assert fa.load_library().fa_last_error()  # a message is set


def test_kvcache_null_seqlens():
    lib = fa.load_library()
    q, k, v, o = good("q"), good("k"), good("v"), good("o")
    st = lib.fa_decode_kvcache(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), None, ctypes.byref(o),
                               None, 0, 0, 0.0, None, 0, None)
    assert st == INVALID


def test_workspace_query_needs_output_pointer():
    lib = fa.load_library()
    q, k, v = good("q"), good("k"), good("v")
    assert lib.fa_fwd_workspace_size(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), 0, 0, None) == INVALID


def test_force_variant_rejects_unknown():
    assert fa.load_library().fa_force_variant(7) == INVALID
    assert fa.load_library().fa_force_variant(0) == OK


def test_stall_hook_rejects_out_of_range_limits():
    lib = fa.load_library()
    assert lib.fa_test_stall_next_call(ctypes.c_ulonglong(0)) == INVALID
    assert lib.fa_test_stall_next_call(ctypes.c_ulonglong(5_000_000_000)) == INVALID


def test_force_tcgen05_form_rejects_unknown():
    lib = fa.load_library()
    assert lib.fa_force_tcgen05_form(4) == INVALID
    assert lib.fa_force_tcgen05_form(-1) == INVALID
    assert lib.fa_force_tcgen05_form(1) == INVALID  # the retired one-tile design
    for form in (fa.TCGEN05_TWO_TILES, fa.TCGEN05_ONE_TILE_MMA, fa.TCGEN05_AUTO):
        assert lib.fa_force_tcgen05_form(form) == OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error():
    q, k, v, o = good("q"), good("k"), good("v"), good("o")
    assert call_fwd(q, k, v, o) == CUDA


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
@pytest.mark.parametrize("dqk,dv", [(8, 8), (32, 32), (40, 40), (80, 80), (96, 96), (112, 112), (160, 128), (160, 160),
                                    (200, 200), (64, 128), (128, 64), (256, 96)])
def test_any_multiple_of_8_head_dims_pass_validation(dqk, dv):
    # validation accepts them; with no device the call then fails on CUDA
    q, k, v, o = desc([1, 1, 8, dqk]), desc([1, 64, 2, dqk]), desc([1, 64, 2, dv]), desc([1, 1, 8, dv])
    assert call_fwd(q, k, v, o) == CUDA


def test_empty_batch_is_a_no_op():
    q, k, v, o = desc([0, 1, 8, 128]), desc([0, 64, 2, 128]), desc([0, 64, 2, 128]), desc([0, 1, 8, 128])
    assert call_fwd(q, k, v, o) == OK


# ------------------------------------------------------------------ work partition

def visible_tiles(n, rb, R, Lq, causal, TK=128, rpc=8):
    """Independent restatement of the tiles a row block needs (bottom-right)."""
    if n <= 0:
        return 0
    rows = range(rb * rpc, min(rb * rpc + rpc, R))
    k = max(min(n, (r % Lq) + n - Lq + 1) if causal else n for r in rows)
    return max(0, math.ceil(max(k, 0) / TK))


CASES = [
    dict(B=1, Lq=1, Hq=32, Hkv=32, Lk=4096, causal=False, seqlens=None, num_ctas=296),
    dict(B=1, Lq=4, Hq=64, Hkv=64, Lk=3000, causal=True, seqlens=None, num_ctas=296),
    dict(B=1, Lq=32, Hq=8, Hkv=2, Lk=128, causal=True, seqlens=None, num_ctas=296),
    dict(B=8, Lq=8, Hq=128, Hkv=128, Lk=16384, causal=True, seqlens=None, num_ctas=296),
    dict(B=64, Lq=1, Hq=32, Hkv=8, Lk=16384, causal=False, seqlens="rand", num_ctas=296),
    dict(B=5, Lq=3, Hq=6, Hkv=2, Lk=100, causal=True, seqlens=[0, 1, 100, 2, 50], num_ctas=7),
    dict(B=3, Lq=1, Hq=2, Hkv=2, Lk=10, causal=False, seqlens=[0, 0, 0], num_ctas=9),
    dict(B=2, Lq=1, Hq=4, Hkv=4, Lk=70000, causal=False, seqlens=None, num_ctas=11),
]


@pytest.mark.parametrize("c", CASES, ids=range(len(CASES)))
@pytest.mark.parametrize("min_share", [1, 2, 5])
@pytest.mark.parametrize("rpc,seg_cost", [(8, 0), (16, 4), (64, 0), (32, 4), (8, 3)])
def test_schedule_covers_balances_and_bounds_partials(c, min_share, rpc, seg_cost):
    c = dict(c)
    if c["seqlens"] == "rand":
        c["seqlens"] = np.random.default_rng(3).integers(1, c["Lk"] + 1, c["B"]).astype(np.int32)
    s = fa.schedule(c["B"], c["Lq"], c["Hq"], c["Hkv"], c["Lk"], c["causal"], c["seqlens"],
                    num_ctas=c["num_ctas"], min_share=min_share, tile_keys=128, rows_per_cta=rpc,
                    seg_cost=seg_cost)
    g = c["Hq"] // c["Hkv"]
    R = g * c["Lq"]
    RB = (R + rpc - 1) // rpc
    want = []
    for b in range(c["B"]):
        n = c["Lk"] if c["seqlens"] is None else int(c["seqlens"][b])
        for rb in range(RB):
            want += [visible_tiles(n, rb, R, c["Lq"], c["causal"], rpc=rpc)] * c["Hkv"]
    tiles = s["unit_tiles"]
    assert tiles.tolist() == want
    # a unit with tiles occupies its tiles, then seg_cost trailing positions
    W = int(tiles.sum()) + seg_cost * int((tiles > 0).sum())
    assert s["work_tiles"] == W
    P = s["ctas_used"]
    assert P == max(1, min(c["num_ctas"], math.ceil(W / min_share)))
    if W == 0:
        assert np.all(s["unit_first_cta"] == -1)
        return
    # P contiguous pieces; the first W % P are one position longer
    share, rem = divmod(W, P)
    starts = [cc * share + min(cc, rem) for cc in range(P)] + [W]
    sizes = np.diff(starts)
    assert np.all(sizes >= 1) and max(sizes) - min(sizes) <= 1
    # each unit's first/last CTA is the one whose piece holds its first/last tile
    has = tiles > 0
    first, last = s["unit_first_cta"][has], s["unit_last_cta"][has]
    pos = 0
    for t, f, l in zip(tiles[has], first, last):
        assert starts[f] <= pos < starts[f + 1]
        assert starts[l] <= pos + int(t) - 1 < starts[l + 1]
        pos += int(t) + seg_cost
    assert pos == W
    assert np.all(np.diff(first) >= 0) and np.all(np.diff(last) >= 0)
    assert first[0] == 0 and (last[-1] == P - 1 or seg_cost > 0)
    # a piece holds at most two partial units (its first and its last segment)
    partial_count = np.zeros(P, dtype=int)
    for f, l in zip(first, last):
        if f != l:
            partial_count[f:l + 1] += 1
    assert partial_count.max(initial=0) <= 2


def test_hld_view_strides():
    x = torch.zeros(32, 4096, 128)
    v = fa.hld_as_blhd(x)
    assert tuple(v.shape) == (1, 4096, 32, 128)
    assert v.stride() == (32 * 4096 * 128, 128, 4096 * 128, 1)


# ------------------------------------------------------------------ paged cache and KV append (host checks)

def call_paged(q, kp, vp, bt=0x20000, bt_stride=4, max_blocks=4, sl=0x30000, o=None):
    lib = fa.load_library()
    o = o or good("o")
    return lib.fa_decode_kvcache_paged(ctypes.byref(q), ctypes.byref(kp), ctypes.byref(vp), ctypes.c_void_p(bt),
                                       bt_stride, max_blocks, ctypes.c_void_p(sl), ctypes.byref(o), None, 0, 0,
                                       0.0, None, 0, None)


@pytest.mark.parametrize("case,expect", [
    ("page_12", UNSUPPORTED), ("page_8", UNSUPPORTED), ("stride_lt_blocks", INVALID), ("null_table", INVALID),
    ("null_seqlens", INVALID), ("blocks_mismatch", INVALID), ("misaligned_table", INVALID),
])
def test_paged_host_validation(case, expect):
    q = good("q")
    kp, vp = desc([10, 16, 2, 128]), desc([10, 16, 2, 128])
    kw = {}
    if case == "page_12":
        kp, vp = desc([10, 12, 2, 128]), desc([10, 12, 2, 128])
    elif case == "page_8":
        kp, vp = desc([10, 8, 2, 128]), desc([10, 8, 2, 128])
    elif case == "stride_lt_blocks":
        kw = dict(bt_stride=2, max_blocks=4)
    elif case == "null_table":
        kw = dict(bt=0)
    elif case == "null_seqlens":
        kw = dict(sl=0)
    elif case == "blocks_mismatch":
        vp = desc([11, 16, 2, 128])
    elif case == "misaligned_table":
        kw = dict(bt=0x20002)
    assert call_paged(q, kp, vp, **kw) == expect
    assert fa.load_library().fa_last_error()


@pytest.mark.parametrize("case", ["shape", "dtype", "heads"])
def test_append_host_validation(case):
    lib = fa.load_library()
    q, k, v, o = good("q"), good("k"), good("v"), good("o")
    kn, vn = desc([1, 1, 2, 128]), desc([1, 1, 2, 128])
    if case == "shape":
        vn = desc([1, 2, 2, 128])
    elif case == "dtype":
        kn = desc([1, 1, 2, 128], dtype=1)
    elif case == "heads":
        kn, vn = desc([1, 1, 4, 128]), desc([1, 1, 4, 128])
    st = lib.fa_decode_kvcache_append(ctypes.byref(q), ctypes.byref(kn), ctypes.byref(vn), ctypes.byref(k),
                                      ctypes.byref(v), None, 0, 0, ctypes.c_void_p(0x30000), ctypes.byref(o), None,
                                      0, 0, 0.0, None, 0, None)
    assert st == INVALID
    assert fa.load_library().fa_last_error()


def test_missing_library_fails_loudly():
    # no fallback: without the built library every call raises (fresh interpreter,
    # the binding pointed at a path that does not exist)
    import subprocess
    import sys

    code = (
        "import torch, decode_flashattention_b200 as fa\n"
        "fa._LIB_PATH = '/nonexistent/libfa_b200.so'\n"
        "q = torch.zeros(1, 1, 8, 128, dtype=torch.float16)\n"
        "k = torch.zeros(1, 64, 2, 128, dtype=torch.float16)\n"
        "try:\n"
        "    fa.fa_fwd(q, k, k)\n"
        "except RuntimeError as e:\n"
        "    print('raised:', e)\n"
        "else:\n"
        "    print('returned')\n"
    )
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert "raised:" in out.stdout and "missing" in out.stdout, out.stdout + out.stderr
