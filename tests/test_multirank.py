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


def _split_worker(rank, world, port, out_dir):
    """A block of mode-0 rows per rank: the rank's share of the state, its
    partial core (a numpy projection of the block standing in for the
    library's, which needs a GPU) and the all-reduce that sums the blocks."""
    import datetime

    import numpy as np
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from rank_sparse_tensor_b200 import split
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shape, ranks = (7, 5, 6), (3, 2, 4)
        rng = np.random.default_rng(0)          # the same whole tensor on every rank
        G = rng.standard_normal(shape) + 1j * rng.standard_normal(shape)
        U = [np.linalg.qr(rng.standard_normal((I, r)) + 1j * rng.standard_normal((I, r)))[0]
             for I, r in zip(shape, ranks)]
        N = G.size
        omega = np.sort(rng.choice(N, size=N // 10, replace=False))
        k = omega.size
        state = {"omega": omega, "U": U, "t": 3, "refreshes": 1, "has_subspace": 1,
                 "core_m": np.arange(2 * np.prod(ranks), dtype=np.float32),
                 "core_v": np.ones(np.prod(ranks), np.float32),
                 "sparse_m": np.arange(2 * k, dtype=np.float32),
                 "sparse_v": np.arange(k, dtype=np.float32)}

        def project(X, Us):
            for n, Un in enumerate(Us):
                X = np.moveaxis(np.tensordot(Un.conj().T, np.moveaxis(X, n, 0), axes=1), 0, n)
            return X

        b0, b1 = split.block_rows(shape[0], world, rank)
        mine = split.block_state(state, shape, b0, b1, cplx=True)
        R = G.reshape(-1).copy()
        R[omega] = 0                           # the residual of the whole tensor
        Rb = R.reshape(shape)[b0:b1]           # this rank's rows
        part = project(Rb, mine["U"])
        core = torch.from_numpy(np.stack([part.real, part.imag], -1).reshape(-1).copy())
        split.allreduce_core(core)
        whole = project(R.reshape(shape), U)
        ref = np.stack([whole.real, whole.imag], -1).reshape(-1)
        with open(os.path.join(out_dir, f"split{rank}.json"), "w") as f:
            json.dump({"rows": [b0, b1], "k": int(mine["k"]),
                       "omega": (mine["omega"] + b0 * 30).tolist(),
                       "sparse_m": mine["sparse_m"].tolist(),
                       "err": float(np.abs(core.numpy() - ref).max() / np.abs(ref).max()),
                       "k_total": int(k), "omega_total": omega.tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_split_blocks_and_core_allreduce_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_split_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"split{r}.json")) for r in range(2)]
    # the blocks tile mode 0 (7 rows: 4 + 3)
    assert res[0]["rows"] == [0, 4] and res[1]["rows"] == [4, 7]
    # every Omega entry lands in exactly one block, in order, with its moments
    assert res[0]["omega"] + res[1]["omega"] == res[0]["omega_total"]
    assert res[0]["k"] + res[1]["k"] == res[0]["k_total"]
    assert res[0]["sparse_m"] + res[1]["sparse_m"] == list(map(float, range(2 * res[0]["k_total"])))
    # the summed partial cores are the whole tensor's core on every rank
    assert res[0]["err"] < 1e-12 and res[1]["err"] < 1e-12


def test_block_rows_cover_mode0():
    sys.path.insert(0, ROOT)
    from rank_sparse_tensor_b200 import split
    for I0 in (1, 7, 256):
        for nb in range(1, min(I0, 9) + 1):
            blocks = [split.block_rows(I0, nb, b) for b in range(nb)]
            assert blocks[0][0] == 0 and blocks[-1][1] == I0
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(nb - 1))
            sizes = [e - b for b, e in blocks]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        split.block_rows(4, 5, 0)
