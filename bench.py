"""Benchmark: achieved K/V HBM bandwidth and time per call of the decode
attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--per-config all|none|names]

One step = one full call of the public API (host plan, split-KV kernel and,
when needed, the LSE combine kernel) over one batch of synthetic input
already resident in HBM.  The headline workload is the largest single-GPU
configuration (MLA-shaped speculative decode, B8 qLen8 H128 192/128,
16384 keys; --workload picks another).  Inputs rotate over enough copies to
exceed 4x the 126 MB L2, so K/V bytes come from HBM.  The K timed steps are
replayed from CUDA graphs (captured calls of the same API) and timed with
CUDA events on the launching stream, a short spin kernel queued ahead so the
host's submission is off the clock; the same graph is replayed again to
give the spread (median, p10, p90) of µs/call.  N > 1 runs independent
replicas (one per GPU) and reports the max time over ranks.

Printed (rank 0, one JSON line): value = algorithmic K/V bytes of all ranks
per second (TB/s); ms_per_step; eager µs/call (calls issued one by one, the
host side of each call on the clock); roofline of the split-KV kernel (the
whole call's time charged to it, with each kernel's isolated CUDA-event
duration for its share); e2e = the same metric through the public API with
pinned host buffers and the host<->device copies inside the timed region;
cpu_baseline = the fp64 oracle on the host cores over a bounded sample; and
per_config = the same measurements for each of the five configurations
C1-C5 (graphs of >= 100 calls, median / p10 / p90 over replays).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
METRIC = "decode attention achieved K/V HBM TB/s (% of B200 peak) and µs/call"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about 2 s worth)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-graph", action="store_true", help="time eager calls instead of graph replays")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="bound of the oracle CPU sample")
    ap.add_argument("--variant", choices=["auto", "mma", "scalar"], default="auto",
                    help="force the split-KV kernel's variant (tensor-core or fp32 FMA)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (a reduced case, e.g. for an ncu capture)")
    ap.add_argument("--reps", type=int, default=10, help="extra replays of the timed graph (µs/call spread)")
    ap.add_argument("--per-config", default="all",
                    help="configurations timed into the per_config block: all (C1-C5), none, or names")
    ap.add_argument("--config-calls", type=int, default=200, help="calls per timed replay of a per_config entry")
    ap.add_argument("--config-reps", type=int, default=11, help="timed replays of a per_config entry")
    ap.add_argument("--config-e2e-steps", type=int, default=2)
    ap.add_argument("--config-cpu-seconds", type=float, default=3.0)
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_init(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist

        dist.barrier(device_ids=[device.index]) if device is not None else dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x0000000000000008: "hw_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000004: "sw_power_cap",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # no NVML: report clocks as unknown
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s)}


# ------------------------------------------------------------------ helpers
def tensor_roofline(w, seqlens, ms_per_call, prof, traffic=None,
                    kernel="tcgen05 dense kernel (whole call)"):
    """Roofline of a prefill-shaped call: bound by the tensor cores.
    achieved = the call's multiply-add flops / its time; peak = the measured
    sustained cuBLAS bf16 rate (the kernel runs back to back for seconds), the
    same for fp16 (the nominal fp16 and bf16 rates are equal)."""
    from decode_flashattention_b200 import workloads as wl

    flops = wl.attn_flops(w, seqlens)
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        peak, kind = float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured (sustained)"
    else:
        peak, kind = 1400.0, "fallback (sustained)"
    achieved = flops / (ms_per_call / 1e3) / 1e12
    iso = {"main": round(prof["main_ms"] / max(prof["main_launches"], 1) * 1e3, 3)}
    if prof.get("combine_ms"):
        iso["combine"] = round(prof["combine_ms"] / max(prof["main_launches"], 1) * 1e3, 3)
    return {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 2),
            "peak": peak, "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "traffic": traffic, "algorithmic_flops_per_launch": flops, "kernel_us": round(ms_per_call * 1e3, 3),
            "isolated_us": iso}


def workload_of(args):
    """The named workload, with its batch size replaced when --batch is given."""
    import dataclasses

    from decode_flashattention_b200 import workloads as wl

    w = wl.WORKLOADS[args.workload or wl.DEFAULT_BENCH]
    if args.batch > 0:
        if w.layout == "hld":
            raise SystemExit("--batch does not apply to the [H, L, D] workloads (B = 1)")
        w = dataclasses.replace(w, B=args.batch)
    return w


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the library's CUDA / C++ sources with comments and whitespace
    removed: it changes when the code does, not when a comment does."""
    import re

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_flashattention_b200", "csrc")
    strip = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, f), encoding="utf-8") as fh:
                text = strip.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", fh.read())
            h.update(f.encode())
            h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the workload's main kernel (split-KV or
    tcgen05) from a committed ncu capture, if it was taken on the current
    kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def cpu_baseline(w, ins, seqlens, seconds: float):
    """The fp64 oracle as it stands, on this host's cores, over a bounded
    sample of the workload's rows; throughput scaled to the same metric.
    ins: (q, k, v) or, for a paged cache, (q, k_pages, v_pages, block_table);
    a paged cache is gathered into its dense form once, untimed, and the
    definition is timed on it."""
    import numpy as np

    import oracle
    from decode_flashattention_b200 import workloads as wl

    oracle.build()
    q = ins[0]
    if w.call == "paged":
        bt = ins[3].cpu().numpy()
        k = oracle.gather_pages(ins[1].cpu(), bt, seqlens.numpy())
        v = oracle.gather_pages(ins[2].cpu(), bt, seqlens.numpy())
    else:
        k, v = ins[1], ins[2]
    cores = os.cpu_count() or 1
    rows_total = w.B * w.Hq * w.Lq
    qc, kc, vc = q.cpu(), None, None
    # estimate: time a handful of rows, then size the sample to the bound
    rng = np.random.default_rng(0)
    all_rows = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.Lq)]
    kc, vc = k.cpu(), v.cpu()
    sl = None if seqlens is None else seqlens.numpy()
    probe = min(rows_total, max(cores, 8))
    idx = rng.choice(rows_total, probe, replace=False)
    t0 = time.perf_counter()
    oracle.attention(qc, kc, vc, causal=w.causal, seqlens=sl, rows=np.array([all_rows[i] for i in idx]),
                     nthreads=cores)
    per_row = (time.perf_counter() - t0) / probe
    n = int(min(rows_total, max(probe, seconds / max(per_row, 1e-9) * 0.8)))
    pick = sorted(rng.choice(rows_total, n, replace=False).tolist()) if n < rows_total else range(rows_total)
    rows = np.array([all_rows[i] for i in pick])
    t0 = time.perf_counter()
    oracle.attention(qc, kc, vc, causal=w.causal, seqlens=sl, rows=rows, nthreads=cores)
    dt = time.perf_counter() - t0
    bytes_sample = wl.kv_bytes(w, seqlens) * (len(rows) / rows_total)
    return {"value": bytes_sample / dt / 1e12, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} of {rows_total} output rows of {w.name} (fp64 C oracle, "
                      f"{dt:.2f} s); K/V bytes scaled by the sampled share of rows",
            "seconds": dt}


# ------------------------------------------------------------------ our arm
class Case:
    """One workload set up on the device: rotating input copies (together
    more than 4x L2, so K/V bytes come from HBM on every call), outputs,
    workspace, and the public call."""

    def __init__(self, w, device, rank, num_splits):
        import torch

        import decode_flashattention_b200 as fa
        from decode_flashattention_b200 import workloads as wl

        self.w = w
        self.device = device
        self.num_splits = num_splits

        def draw(seed):
            if w.call == "paged":
                q, kp, vp, bt, sl = wl.make_paged_inputs(w, device, seed=seed)
                return (q, kp, vp, bt), sl
            q, k, v, sl = wl.make_inputs(w, device, seed=seed)
            return (q, k, v), sl

        self.ins0, self.sl0 = draw(w.seed + 1000 * rank)
        q0 = self.ins0[0]
        self.per_copy = sum(t.numel() * t.element_size() for t in self.ins0)
        self.n_copies = max(1, math.ceil(4 * L2_BYTES / max(self.per_copy, 1)))
        self.copies = [self.ins0] + [draw(w.seed + 1000 * rank + c)[0] for c in range(1, self.n_copies)]
        self.sl_dev = self.sl0.to(device) if self.sl0 is not None else None
        self.outs = [wl.empty_output(w, q0) for _ in range(self.n_copies)]
        self.lses = [torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=device)
                     for _ in range(self.n_copies)]
        if w.call == "paged":
            ws_bytes = fa.paged_workspace_size(q0, self.ins0[1], self.ins0[2], self.ins0[3].shape[1], num_splits)
        elif w.call == "kvcache":
            ws_bytes = fa.kvcache_workspace_size(*self.ins0, num_splits)
        else:
            ws_bytes = fa.fwd_workspace_size(*self.ins0, w.causal, num_splits)
        self.ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)
        self.bytes_per_step = wl.kv_bytes(w, self.sl0)
        self.flops_per_step = wl.attn_flops(w, self.sl0)

    def call(self, ins, sl, o, l):
        import decode_flashattention_b200 as fa

        w, ns, ws = self.w, self.num_splits, self.ws
        if w.call == "paged":
            return fa.fa_decode_kvcache_paged(*ins, sl, causal=w.causal, num_splits=ns, out=o, lse=l, workspace=ws)
        if w.call == "kvcache":
            return fa.fa_decode_kvcache(*ins, sl, causal=w.causal, num_splits=ns, out=o, lse=l, workspace=ws)
        return fa.fa_fwd(*ins, causal=w.causal, num_splits=ns, out=o, lse=l, workspace=ws)

    def step(self, i):
        c = i % self.n_copies
        self.call(self.copies[c], self.sl_dev, self.outs[c], self.lses[c])

    def graphs(self, K):
        """CUDA graphs replaying K calls of the public API (chunks of at most
        2000 calls); returns (graphs, our kernel launches they hold)."""
        import torch

        import decode_flashattention_b200 as fa

        out, launches, done = [], 0, 0
        while done < K:
            n = min(2000, K - done)
            n0 = fa.launch_count()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(done, done + n):
                    self.step(i)
            launches += fa.launch_count() - n0
            out.append(g)
            done += n
        for g in out:  # warm the graphs themselves
            g.replay()
        torch.cuda.synchronize()
        return out, launches


def lead_sleep():
    """Queue ~0.2 ms of device work ahead of a timed region, so the host has
    submitted the region's work before its first event fires: the events then
    time the device, not the host's launch latency."""
    import torch

    torch.cuda._sleep(int(4e5))


def replay_ms(graphs, stream):
    """Device time of one replay of `graphs` (CUDA events on the stream)."""
    import torch

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lead_sleep()
    e0.record(stream)
    for g in graphs:
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def pct(xs, q):
    xs = sorted(xs)
    if not xs:
        return None
    i = min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))
    return xs[i]


def e2e_measure(case, E, world, device):
    """The metric through the public API from pinned host buffers: every step
    copies its inputs host -> device, calls, and copies O and lse back."""
    import torch

    w = case.w

    def pinned_like(t):
        # the device tensor's own layout ([H, L, D] storage stays [H, L, D]),
        # so each copy is one plain memcpy of the storage
        h = torch.empty_strided(t.size(), t.stride(), dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    hins = [pinned_like(t) for t in case.ins0]
    hsl = case.sl0.pin_memory() if case.sl0 is not None else None
    o0, l0 = case.outs[0], case.lses[0]
    ho = torch.empty_strided(o0.size(), o0.stride(), dtype=w.dtype, pin_memory=True)
    hl = torch.empty_strided(l0.size(), l0.stride(), dtype=torch.float32, pin_memory=True)
    dins = [torch.empty_like(t) for t in case.ins0]
    dsl = torch.empty_like(case.sl_dev) if case.sl_dev is not None else None
    h2d = sum(t.numel() * t.element_size() for t in hins) + (hsl.numel() * 4 if hsl is not None else 0)
    d2h = ho.numel() * ho.element_size() + hl.numel() * 4
    stream = torch.cuda.current_stream(device)

    def e2e_step():
        for d, h in zip(dins, hins):
            d.copy_(h, non_blocking=True)
        if dsl is not None:
            dsl.copy_(hsl, non_blocking=True)
        o, l = case.call(dins, dsl, o0, l0)
        ho.copy_(o, non_blocking=True)
        hl.copy_(l, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world, device)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(E):
        e2e_step()
    x1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(x0.elapsed_time(x1), world, device)
    total = sum_over_ranks(case.bytes_per_step * E, world, device)
    del dins, hins
    return {"value": round(total / (ms / 1e3) / 1e12, 5), "unit": "TB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": E, "ms_per_step": ms / E}


def isolated_kernels(case, Kb):
    """Each kernel's own duration: the library brackets its launches with CUDA
    events on the call's stream (and launches them without programmatic
    overlap, so each event pair times one kernel alone).  A spin kernel ahead
    of the calls lets the host queue them all before the first runs, so no
    host launch gap falls between an event and its kernel."""
    import torch

    import decode_flashattention_b200 as fa

    fa.profile_enable(True)
    torch.cuda._sleep(int(40e6))  # about 20 ms of device time
    for i in range(Kb):
        case.step(i)
    torch.cuda.synchronize()
    prof = fa.profile_read()
    fa.profile_enable(False)
    fa.check_status()
    return prof


def hbm_roofline(case, us_per_call, prof, peak, peak_kind, traffic):
    b = case.bytes_per_step
    achieved = b / (us_per_call / 1e6) / 1e9
    main_iso = prof["main_ms"] / max(prof["main_launches"], 1)
    comb_iso = prof["combine_ms"] / max(prof["main_launches"], 1)  # per step (0 when no combine ran)
    share_main = main_iso / (main_iso + comb_iso) if main_iso + comb_iso > 0 else 1.0
    return {
        "bound": "hbm",
        "kernel": "split-KV kernel, charged with the whole call (combine and boundaries included)",
        "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
        "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes_per_launch": b,
        "kernel_us": round(us_per_call, 3),
        "duration_method": "CUDA events on the launching stream around the timed region / calls (whole call)",
        "share": round(share_main, 4),
        "isolated_us": {"splitkv": round(main_iso * 1e3, 3),
                        "combine": round(prof["combine_ms"] / max(prof["combine_launches"], 1) * 1e3, 3)},
        "isolated_launches": prof["main_launches"],
    }


def config_entry(w, world, rank, device, args, reuse=None):
    """Per-config block: µs/call (median, p10, p90 over repeated timed
    replays of a graph of >= 100 calls), TB/s, fraction of the measured peak,
    ncu traffic, e2e and the oracle's CPU baseline."""
    import torch

    import decode_flashattention_b200 as fa

    case = reuse if reuse is not None else Case(w, device, rank, args.num_splits)
    for i in range(3):
        case.step(i)
    torch.cuda.synchronize()
    fa.check_status()
    dispatch = fa.last_dispatch()
    stream = torch.cuda.current_stream(device)
    calls = max(100, args.config_calls)
    graphs, _ = case.graphs(calls)
    reps = []
    for _ in range(max(3, args.config_reps)):
        barrier(world, device)
        reps.append(max_over_ranks(replay_ms(graphs, stream), world, device) / calls * 1e3)
    fa.check_status()
    del graphs
    med = pct(reps, 0.5)
    peak, peak_kind = peaks()
    tbs = case.bytes_per_step / (med / 1e6) / 1e12
    ent = {
        "workload": w.name, "description": w.description,
        "us_per_call": round(med, 3), "us_p10": round(pct(reps, 0.1), 3), "us_p90": round(pct(reps, 0.9), 3),
        "calls_per_rep": calls, "reps": len(reps),
        "value": round(tbs * world, 4), "unit": "TB/s", "frac": round(tbs * 1e3 / peak, 4), "peak": peak,
        "peak_kind": peak_kind, "kv_bytes_per_call": case.bytes_per_step,
        "query_tokens_per_s": round(w.B * w.Lq * world / (med / 1e6), 1),
        "traffic": recorded_traffic(w.name),
        "dispatch": {k: dispatch[k] for k in ("variant", "grid", "rows_per_cta", "units", "combine_launched")},
    }
    if dispatch.get("variant") == fa.VARIANT_TCGEN05 or w.name == "gqa_prefill_fp16":
        ent["note"] = "latency-bound (64 KB of K/V): parity and µs/call only" if w.name == "gqa_prefill_fp16" else None
    ent["e2e"] = e2e_measure(case, max(1, args.config_e2e_steps), world, device)
    ent["cpu_baseline"] = (cpu_baseline(w, case.ins0, case.sl0, args.config_cpu_seconds)
                           if world == 1 else None)
    if reuse is None:
        del case
        torch.cuda.empty_cache()
    return ent


def run_ours(args):
    import torch

    import decode_flashattention_b200 as fa
    from decode_flashattention_b200 import workloads as wl

    world, rank, local = dist_init(args)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    fa.load_library()
    fa.force_variant({"auto": fa.VARIANT_AUTO, "mma": fa.VARIANT_MMA, "scalar": fa.VARIANT_SCALAR}[args.variant])
    name = args.workload or wl.DEFAULT_BENCH
    w = workload_of(args)
    case = Case(w, device, rank, args.num_splits)
    stream = torch.cuda.current_stream(device)
    W = max(args.warmup, 3)
    for i in range(W):
        case.step(i)
    torch.cuda.synchronize()
    fa.check_status()
    dispatch = fa.last_dispatch()

    # steps: about 2 s of work unless given
    if args.steps > 0:
        K = args.steps
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(20):
            case.step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        per = e0.elapsed_time(e1) / 20 / 1e3
        K = int(max_over_ranks(int(min(200000, max(50, 2.0 / max(per, 1e-7)))), world, device))

    # --- the timed region: exactly K calls, replayed from CUDA graphs of the
    # public call, device time by CUDA events on the launching stream --------------
    use_graph = not args.no_graph
    if use_graph:
        graphs, launches = case.graphs(K)
    sampler = ClockSampler(device.index)
    with sampler:
        barrier(world, device)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if use_graph:
            lead_sleep()
            e0.record(stream)
            for g in graphs:
                g.replay()
        else:
            n0 = fa.launch_count()
            e0.record(stream)
            for i in range(K):
                case.step(i)
            launches = fa.launch_count() - n0
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
        ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        # the same K calls replayed again: the spread of µs/call over replays
        reps = []
        if use_graph:
            for _ in range(max(3, args.reps)):
                barrier(world, device)
                reps.append(max_over_ranks(replay_ms(graphs, stream), world, device) / K * 1e3)
    fa.check_status()
    if use_graph:
        del graphs

    # --- eager calls: the host side of each call (validation, plan, two tensor-map
    # encodes, launches) is on the clock -------------------------------------------
    Ke = min(K, 200)
    barrier(world, device)
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for i in range(Ke):
        case.step(i)
    x1.record(stream)
    torch.cuda.synchronize()
    eager_ms = max_over_ranks(x0.elapsed_time(x1), world, device)
    # the host's own cost per call, with the device kept busy by a spin kernel
    # queued first so the host never waits on it
    torch.cuda._sleep(int(Ke * 2e5))  # ~0.1 ms of device time per call
    t0 = time.perf_counter()
    for i in range(Ke):
        case.step(i)
    host_s = time.perf_counter() - t0
    torch.cuda.synchronize()
    fa.check_status()

    prof = isolated_kernels(case, int(min(K, 200)))
    e2e = e2e_measure(case, max(1, args.e2e_steps), world, device)

    total_bytes = sum_over_ranks(case.bytes_per_step * K, world, device)
    value = total_bytes / (ms / 1e3) / 1e12
    peak, peak_kind = peaks()
    tc = dispatch.get("variant") == fa.VARIANT_TCGEN05 or w.tensor_bound
    us_call = ms / K * 1e3
    traffic = recorded_traffic(name) if not args.batch else None
    clocks = sampler.summary()
    # Roofline of the call.  Both kernels run back to back with programmatic
    # overlap, so no event pair can time one of them inside the timed region
    # without breaking that overlap; the achieved figure therefore charges the
    # split-KV kernel with the whole time per call (its combine and both kernel
    # boundaries included) -- a lower bound on its own bandwidth.  The isolated
    # per-kernel event times give the kernels' shares, reported beside it (the
    # ncu launch list of the same command gives the same shares).
    roof = (tensor_roofline(w, case.sl0, ms / K, prof, traffic,
                            "tcgen05 dense kernel (whole call)" if dispatch.get("variant") == fa.VARIANT_TCGEN05
                            else "split-KV kernel + combine (whole call)") if tc
            else hbm_roofline(case, us_call, prof, peak, peak_kind, traffic))
    cpu = cpu_baseline(w, case.ins0, case.sl0, args.cpu_seconds) if world == 1 else None

    # --- every configuration of the metric, each timed the same way -------------------
    per_config = {}
    if args.per_config != "none":
        names = wl.CONFIGS if args.per_config == "all" else args.per_config.split(",")
        for cname in names:
            wc = wl.WORKLOADS[cname]
            key = next((k for k, v in wl.CONFIG_IDS.items() if v == cname), cname)
            if cname == name and not args.batch:
                per_config[key] = config_entry(wc, world, rank, device, args, reuse=case)
            else:
                per_config[key] = config_entry(wc, world, rank, device, args)
    if rank != 0:
        return
    res = {
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "TB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms / K,
        "us_per_call": us_call,
        "us_per_call_replays": {"median": round(pct(reps, 0.5), 3) if reps else None,
                                "p10": round(pct(reps, 0.1), 3) if reps else None,
                                "p90": round(pct(reps, 0.9), 3) if reps else None,
                                "replays": len(reps), "calls_per_replay": K},
        "eager": {"us_per_call": round(eager_ms / Ke * 1e3, 3), "calls": Ke,
                  "host_us_per_call": round(host_s / Ke * 1e6, 3),
                  "what": "calls issued one by one from Python through the C ABI (host validation, plan, "
                          "two tensor-map encodes and the launches of each call on the clock): device time "
                          "per call, and the host's own time per call measured while the device is kept busy"},
        "pct_of_peak_per_gpu": round(100 * value / world * 1e3 / peak, 2),
        "query_tokens_per_s": round(wl.tokens_per_call(w) * K * world / (ms / 1e3), 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16" if w.dtype == torch.float16 else "bf16",
        "data": "synthetic: Q/K/V i.i.d. N(0,1), seeded; no dataset or weights",
        "config": {
            "workload": name, "description": w.description, "call": w.call, "layout": w.layout,
            "batch_override": args.batch or None,
            "B": w.B, "Lq": w.Lq, "Hq": w.Hq, "Hkv": w.Hkv, "Lk": w.Lk, "Dqk": w.Dqk, "Dv": w.Dv,
            "causal": w.causal, "num_splits": args.num_splits or "auto", "variant": args.variant,
            "kv_bytes_per_step": case.bytes_per_step,
            "l2": f"inputs rotate over {case.n_copies} copies ({case.n_copies * case.per_copy / 1e6:.0f} MB > 4x L2)",
            "launch": "cuda_graph_replay" if use_graph else "eager",
            "timing": "device time by CUDA events on the launching stream; a short spin kernel queued ahead of "
                      "each timed region so the host's submission is off the clock",
            "parallelism": f"replicas{world}" if world > 1 else "single_gpu",
            "dispatch": dispatch,
        },
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "cpu_baseline": cpu,
        "per_config": per_config,
    }
    print(json.dumps(res), flush=True)


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    from decode_flashattention_b200 import workloads as wl

    name = args.workload or wl.DEFAULT_BENCH
    w = workload_of(args)
    if w.call == "paged":
        q, kp, vp, bt, sl = wl.make_paged_inputs(w, "cpu")
        ins = (q, kp, vp, bt)
    else:
        q, k, v, sl = wl.make_inputs(w, "cpu")
        ins = (q, k, v)
    W = max(args.warmup, 3)
    K = args.steps if args.steps > 0 else 3
    per_step = max(1.0, min(args.cpu_seconds, 60.0 / max(K + W, 1)))
    for _ in range(min(W, 1)):
        cpu_baseline(w, ins, sl, per_step / 4)
    vals, secs = [], 0.0
    for _ in range(K):
        r = cpu_baseline(w, ins, sl, per_step)
        vals.append(r["value"])
        secs += r["seconds"]
    value = sum(vals) / len(vals)
    res = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": world,
           "steps": K, "warmup": W, "ms_per_step": secs / K * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic: Q/K/V i.i.d. N(0,1), seeded; no dataset or weights",
           "config": {"workload": name, "description": w.description},
           "cpu_baseline": {"value": value, "unit": "TB/s", "cores": r["cores"], "kind": "oracle",
                            "sample": r["sample"]},
           "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    try:
        import torch.distributed as dist

        if dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
