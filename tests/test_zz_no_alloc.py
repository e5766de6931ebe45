"""fa_decode_kvcache_noalloc: the KV-cache decode call for callers that cannot
allocate device memory (a serving-runtime plugin whose host owns all device
memory, or a decode loop that must not risk cudaMalloc's implicit
synchronisation).  It takes its split-KV scratch from a fixed array compiled
into the library instead of a caller workspace.

The test calls it through the C ABI twice in a row, on different inputs, and
checks each result against the fp64 oracle and against the regular
fa_decode_kvcache (caller workspace), both within the parity tolerances; a
request needing more scratch than the array holds must be refused with a
message.  This file is named to be collected
last, and it runs the same way alone in a fresh process.
"""
import ctypes

import pytest
import torch

import decode_flashattention_b200 as fa
from decode_flashattention_b200 import FaTensor
from decode_flashattention_b200 import workloads as wl

from helpers import compare, oracle_full

pytestmark = pytest.mark.gpu

UNSUPPORTED = 2


def _lib():
    lib = fa.load_library()
    fn = lib.fa_decode_kvcache_noalloc
    T = ctypes.POINTER(FaTensor)
    fn.restype = ctypes.c_int
    fn.argtypes = [T, T, T, ctypes.c_void_p, T, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                   ctypes.c_float, ctypes.c_void_p]
    lib.fa_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return lib


def _desc(t):
    d = FaTensor()
    d.data = t.data_ptr()
    d.dtype = 0 if t.dtype == torch.float16 else 1
    for i in range(4):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _noalloc(lib, q, k, v, sl, causal, num_splits=0):
    o = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[3], dtype=q.dtype, device=q.device)
    lse = torch.empty(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = lib.fa_decode_kvcache_noalloc(_desc(q), _desc(k), _desc(v), ctypes.c_void_p(sl.data_ptr()),
                                       _desc(o), ctypes.c_void_p(lse.data_ptr()), num_splits, int(causal),
                                       0.0, ctypes.c_void_p(stream))
    return st, o, lse


CASES = [
    wl.Workload("noalloc_a", "kvcache", "blhd", torch.bfloat16, B=8, Lq=1, Hq=32, Hkv=8, Lk=4096,
                Dqk=128, Dv=128, causal=False, seed=301, seqlen_lo=1, seqlen_hi=4096),
    wl.Workload("noalloc_b", "kvcache", "blhd", torch.float16, B=3, Lq=4, Hq=16, Hkv=4, Lk=2500,
                Dqk=128, Dv=128, causal=True, seed=302, seqlen_lo=0, seqlen_hi=2500),
]


def test_noalloc_matches_regular_call_twice_in_a_row():
    lib = _lib()
    assert lib.fa_noalloc_scratch_bytes() == 8 << 20
    for w in CASES:
        q, k, v, sl = wl.make_inputs(w, "cuda")
        sl = sl.cuda()
        st, o, lse = _noalloc(lib, q, k, v, sl, w.causal)
        assert st == 0, lib.fa_last_error()
        ro, rl = fa.fa_decode_kvcache(q, k, v, sl, causal=w.causal)
        torch.cuda.synchronize()
        fa.check_status()
        eo, el = oracle_full(q, k, v, w.causal, seqlens=sl)
        compare(o.float().cpu().numpy(), lse.cpu().numpy(), eo, el, w.dtype, w.name + " vs oracle")
        compare(o.float().cpu().numpy(), lse.cpu().numpy(), ro.float().cpu().numpy(), rl.cpu().numpy(),
                w.dtype, w.name + " vs fa_decode_kvcache")


def test_noalloc_refuses_scratch_beyond_its_array():
    lib = _lib()
    w = CASES[0]
    q, k, v, sl = wl.make_inputs(w, "cuda")
    st, _, _ = _noalloc(lib, q, k, v, sl.cuda(), False, num_splits=4096)
    assert st == UNSUPPORTED
    assert b"scratch" in lib.fa_last_error()
