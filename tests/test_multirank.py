"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each
rank steps its own tensors, the job time is the slowest rank's, the job
throughput counts every rank's elements, rank 0 alone reports; and the
reference arm under a 2-rank launch prints once and exits 0 on every rank."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
torch = pytest.importorskip("torch")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, loc = bench.rank_env()
        seeds = bench.tensor_seeds(r, 4)
        # a rank-dependent "measured" time: rank 1 is the slower one
        my_ms = 100.0 + 50.0 * r
        mx = bench.max_over_ranks(my_ms, w)
        value = bench.job_throughput(w, 1000, 10, mx)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"world": w, "rank": r, "local": loc, "seeds": seeds, "max_ms": mx,
                       "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [x["rank"] for x in res] == [0, 1] and all(x["world"] == 2 for x in res)
    # every rank holds the slowest time
    assert res[0]["max_ms"] == res[1]["max_ms"] == 150.0
    # whole-job throughput: 2 ranks x 1000 elements x 10 steps / 0.15 s
    assert res[0]["value"] == pytest.approx(2 * 1000 * 10 / 0.15)
    # independent problems: no seed shared between ranks
    s0 = {tuple(x) for x in res[0]["seeds"]}
    s1 = {tuple(x) for x in res[1]["seeds"]}
    assert s0.isdisjoint(s1) and len(s0) == len(s1) == 4


def test_single_rank_defaults(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 10, 2, 1000.0) == 20.0


def test_reference_arm_two_ranks():
    """`bench.py --impl reference` launched on 2 ranks: rank 0 prints one JSON
    line with impl=reference, rank 1 does no work and exits 0."""
    port = _free_port()
    env = dict(os.environ, TGD_ORACLE_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--workload", "fno_c64_64x64x32x17"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
