"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the
barrier, max-over-ranks timing and the whole-job throughput; and the
reference arm under torchrun (rank 0 prints one JSON line, other ranks exit
0 without work).  Sessions are independent replicas, so no collective
touches the data path."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_pg(world, "gloo")
    bench.barrier(world)
    elapsed = 100.0 + 50.0 * rank            # rank 1 is the slow one
    m = bench.max_over_ranks(elapsed, world)
    v = bench.aggregate_throughput(10, m, world)
    q.put((rank, m, v))
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world, port = 2, 29731
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in got:
        assert m == 150.0                        # both ranks see the slowest rank's time
        assert abs(v - 2 * 10 / 0.150) < 1e-9    # all ranks' steps over that time


@pytest.mark.slow
def test_reference_arm_under_torchrun():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29733", "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                      # rank 0 only
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0
    # the line carries every key of the bench contract, with our arm's metric and unit
    sys.path.insert(0, ROOT)
    import bench
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in j, key
    assert j["metric"] == bench.METRIC and j["unit"] == bench.UNIT
    assert j["higher_is_better"] is True and j["steps"] == 1 and j["warmup"] == 3
    assert j["config"]["workload"] == bench.WORKLOAD
    for key in ("value", "unit", "cores", "kind", "sample"):
        assert key in j["cpu_baseline"], key
    assert j["cpu_baseline"]["value"] == j["value"] and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
