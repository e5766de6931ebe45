"""The bench's multi-rank plumbing on CPU: two gloo ranks, as torchrun would
start them, each timing an independent replica.

Checks that the reported time is the max over ranks, the reported volume the
sum over ranks, that the barrier releases both ranks, and that the reference
arm prints exactly one JSON line from rank 0 only while the other rank exits
without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cpu = torch.device("cpu")
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world, cpu)
        v = bench.sum_over_ranks(100.0 * (rank + 1), world, cpu)
        bench.barrier(world)
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


def test_max_and_sum_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    # every rank sees the slowest rank's time and the total volume
    assert res[0] == res[1] == (15.0, 300.0)


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.sum_over_ranks(2.0, 1, None) == 2.0


def _reference_arm(rank, world, port):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
               WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "gqa_prefill_fp16", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.2", "--gpus", str(world)]
    return subprocess.Popen(cmd, env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_line_from_rank0_only():
    port = _free_port()
    procs = [_reference_arm(r, 2, port) for r in range(2)]
    outs = [p.communicate(timeout=240) for p in procs]
    assert [p.returncode for p in procs] == [0, 0], [o[1][-2000:] for o in outs]
    lines0 = [l for l in outs[0][0].splitlines() if l.strip()]
    lines1 = [l for l in outs[1][0].splitlines() if l.strip()]
    assert lines1 == []
    assert len(lines0) == 1
    rec = json.loads(lines0[0])
    assert rec["impl"] == "reference"
    assert rec["n_gpus"] == 2 and rec["steps"] == 1 and rec["warmup"] == 3
    assert rec["value"] > 0 and rec["unit"] == "TB/s" and rec["higher_is_better"] is True
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["e2e"] == {"value": rec["value"], "unit": "TB/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert rec["config"]["workload"] == "gqa_prefill_fp16"
