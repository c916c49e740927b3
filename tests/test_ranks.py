"""The multi-rank host logic of bench.py on CPU: two `gloo` ranks run the
barrier, the max-over-ranks reduction of a timed region and the whole-job
aggregate that `bench.py --gpus N` uses under NCCL; the reference arm prints
from rank 0 only.  No GPU is needed."""

import json
import os
import socket
import subprocess
import sys

import pytest

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank             # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, world)
        rate = bench.whole_job_rate(units_per_rank=8192, world=world, steps=4, total_ms=total)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump({"total": total, "rate": rate}, f)


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_rate(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    for g in got:
        assert g["total"] == 15.0                              # the slowest rank's time, on every rank
        assert g["rate"] == pytest.approx(8192 * 2 * 4 / 0.015)  # all ranks' units / that time


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(1)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 10, 1000.0) == pytest.approx(1000.0)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_from_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), ORACLE_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "prefill_512", "--steps", "1", "--warmup", "1", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank != 0:
        assert lines == []
        return
    line = json.loads(lines[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
