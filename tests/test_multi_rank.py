"""Multi-process logic of bench.py on CPU (gloo, world size 2).

The method needs no exchange between GPUs ("replicas only"): each rank runs its
own replica and the only collectives are barriers and the max over ranks of the
timing.  These tests run that logic with two gloo ranks on the host.
"""

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 2.0 + rank  # the slower rank decides
        m = bench.max_over_ranks(ms, torch.device("cpu"))
        dist.barrier()
        out[rank] = (m, bench.job_value(world, 1e12, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = 29500 + os.getpid() % 1000
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == out[1]
        m, v = out[0]
        assert m == 3.0
        assert v == pytest.approx(2 * 1e12 / 3e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.max_over_ranks(1.5, torch.device("cpu")) == 1.5


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--gpus", "2"], capture_output=True, text=True, env=env, timeout=300)
    assert p.returncode == 0, p.stderr
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
