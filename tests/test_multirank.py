"""The bench's multi-rank logic on CPU: two gloo ranks (one process each).

On GPUs every rank owns its own layer instances (replicas, weak scaling, no
data-path collective); the only collective is the all-reduce MAX of the
timed region, and rank 0 alone prints.  Here the same helpers run with the
gloo backend: the slowest rank's time reaches every rank, the whole-job
value counts every rank's bytes, the ranks' synthetic layers differ, and
the reference arm leaves ranks other than 0 without work.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        slowest = bench.max_over_ranks(my_ms, world)
        shape = synth.workloads()["llama7b-q-4bit"][0]
        small = synth.Shape(shape.name, 64, 256, shape.bits, shape.density, 1)
        layer = synth.layer_for(small, instance=bench.instance_id(rank, 0))
        x = synth.x_for(small, instance=bench.instance_id(rank, 0))
        # reference arm on a rank other than 0: returns at once, prints nothing
        ref_rc = None
        if rank != 0:
            import argparse

            ref_rc = bench.run_reference(argparse.Namespace(workload="llama7b-q-4bit", shape_index=0, steps=1,
                                                            warmup=0, gpus=world, csr="balanced"))
        dist.barrier()
        out[rank] = (slowest, bench.whole_job_gbs(world, 1_000_000, 10, slowest), int(layer.codes[0, 0]),
                     int(x[0, 0]), ref_rc)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_own_different_layers():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # whole job: both ranks' bytes over the slowest rank's time
    assert res[0][1] == pytest.approx(2 * 1_000_000 * 10 / 0.015 / 1e9)
    # replicas: each rank draws its own layer and activations
    assert (res[0][2], res[0][3]) != (res[1][2], res[1][3])
    assert res[1][4] == 0


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_gbs(1, 2_000_000, 4, 8.0) == pytest.approx(2_000_000 * 4 / 0.008 / 1e9)
    assert bench.instance_id(0, 3) != bench.instance_id(1, 3)


def test_gpus_flag_spawns_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself (here in
    the CPU self-test mode: gloo, fixed per-rank times): rank 0 alone prints,
    n_gpus is the real world size and the time is the slowest rank's."""
    import json
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "10",
                          "--selftest-ranks"], capture_output=True, text=True, timeout=180, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2
    assert rec["ms"] == 20.0
    assert rec["value"] == pytest.approx(2 * 1_000_000 * 10 / 0.020 / 1e9)


def test_bench_step_is_a_stack_of_layers_larger_than_l2():
    sys.path.insert(0, ROOT)
    import bench

    l2 = 126 * 1024 * 1024
    # the 18.4 MB bench layer: 32 layers (590 MB) already exceed 4x L2
    assert bench.stack_depth(l2, 18_376_054) == 32
    # the 9 MB 4096x4096 4-bit layer needs more than 32 to reach 4x L2
    r = bench.stack_depth(l2, 9_004_678)
    assert r > 32 and r * 9_004_678 >= 4 * l2
    assert bench.graph_plan(20, 16) == (1, 4)
    assert bench.graph_plan(32, 16) == (2, 0)
