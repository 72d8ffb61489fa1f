"""World-size-2 checks (gloo, CPU) of the benchmark's multi-rank host logic.

The operator shards by (sequence, head) with no exchange step, so N GPUs run
independent replicas; the only cross-rank logic is the timing reduction (max
over ranks) and the whole-job aggregate.  These run without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["KDA_ROOT"])
import datetime
import torch.distributed as dist
import bench
rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
mine = [3.0, 7.5][rank]
m = bench.max_over_ranks(mine, world)
rate = bench.aggregate_rate(1000.0, world, m)
dist.barrier()
print(json.dumps({"rank": rank, "max": m, "rate": rate}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_and_aggregate_with_two_gloo_ranks(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), KDA_ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(out.strip().splitlines()[-1])
    import json
    res = [json.loads(o) for o in outs]
    for r in res:
        assert r["max"] == 7.5                       # both ranks see the slowest rank's time
        assert abs(r["rate"] - 2 * 1000.0 / 7.5e-3) < 1e-6   # units of all ranks / max time


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.aggregate_rate(131072, 1, 50.0) == pytest.approx(131072 / 0.05)


def test_reference_arm_other_ranks_exit_without_work():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        T, steps, warmup, gpus = 131072, 1, 0, 2
    # rank 1 of 2 returns immediately (rank 0 alone runs the oracle and prints)
    assert bench.main_reference(A(), 1, 2) is None
