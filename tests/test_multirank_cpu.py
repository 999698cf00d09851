"""The bench's multi-rank host logic on CPU: two gloo ranks (the layer shards only as
independent replicas, so the only cross-rank steps are the barrier and the max-over-ranks
timing).  No GPU."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [120.0, 150.0][rank]                    # rank 1 is the slow one
    ms = bench.max_over_ranks_(local_ms, world, "cpu")
    value = bench.job_throughput(8192, 20, world, ms)
    dist.barrier()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"ms": ms, "value": value}, f)
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo(tmp_path):
    port = 29500 + os.getpid() % 1000
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert res[0]["ms"] == res[1]["ms"] == 150.0
    assert res[0]["value"] == pytest.approx(2 * 8192 * 20 / 0.150)


def test_reference_arm_prints_on_rank0_only():
    """`bench.py --impl reference` under two ranks: rank 0 prints one JSON line (the oracle
    on the toy layer), rank 1 exits 0 without work."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--workload", "toy", "--steps", "1", "--warmup", "0"],
                        capture_output=True, text=True, env=env, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0", WORLD_SIZE="1")
    r0 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--workload", "toy", "--steps", "1", "--warmup", "0"],
                        capture_output=True, text=True, env=env, timeout=300)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
