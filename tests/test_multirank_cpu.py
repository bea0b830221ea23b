"""The multi-rank logic of bench.py on CPU with the gloo backend (world size 2):
every rank takes the same collective steps, timing is the maximum over ranks,
and the reference arm runs on rank 0 alone.  The units of the attention path
are independent, so N GPUs run N replicas with no data-path collective; these
tests cover the plumbing around that, not a GPU kernel."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    from exact_io_aware_52_b200 import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        slowest = bench.max_over_ranks(1.5 + rank, world, device="cpu")
        cfg = bench.workload_config(workloads.WORKLOADS[4], world, 403 * 10**6)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "parallelism": cfg["parallelism"]}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo(tmp_path):
    port = 29500 + (os.getpid() % 1000)
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        rec = json.load(open(tmp_path / f"rank{rank}.json"))
        assert rec["slowest"] == 2.5            # both ranks see the slowest rank's time
        assert rec["parallelism"] == "replicas x2"


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        rec = json.loads(lines[0])
        assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["higher_is_better"]
        assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
