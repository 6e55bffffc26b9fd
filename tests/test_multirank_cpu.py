"""The N>1 benchmark path on CPU: two gloo ranks (no GPU).

Each rank times its own batch (weak scaling, no collective on the data path);
the job's time is the maximum over ranks and its rate counts every rank's
units.  The reference arm under a multi-rank launch runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(times[rank], world)
        out[rank] = (m, bench.job_throughput(10.0, world, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_with_two_gloo_ranks():
    world, port = 2, _free_port()
    times = [3.0, 5.0]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        m, rate = res[r]
        assert m == 5.0
        assert rate == pytest.approx(world * 10.0 / 5e-3)


def test_reference_arm_only_rank0_prints_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert '"impl": "reference"' in lines[0]


def test_stage_model_matches_launches_per_call():
    """The benchmark's per-launch byte model lists one entry per kernel the library launches,
    for every path and reading (int8 x adds its pass in front)."""
    import bench
    from group_wise_int8_b200 import synth, wino
    layer = synth.workload("resnet18")[0]
    shape = (layer.N, layer.H, layer.W, layer.Cin, layer.Cout)
    for y_path in (wino.YPATH_RECOMPUTE, wino.YPATH_Y32):
        for x_int8 in (False, True):
            plan = wino.Plan(layer.m, layer.points, None, None, layer.group, y_path=y_path, x_int8=x_int8)
            model = bench.stage_model(layer, plan.resolved_config(*shape)[0], x_int8)
            assert len(model) == plan.launches_per_call(*shape)
            assert (model[0][0] == "input_quant") == x_int8
            assert all(nbytes > 0 for _, nbytes, _ in model)
