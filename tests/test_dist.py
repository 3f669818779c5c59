"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (no GPU).

The lookup is per token, so ranks shard tokens with the tables replicated and
no data-path collective; the only collectives are the barrier and the
max-over-ranks of the timing.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import datetime

    import bench
    import oracle
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs

    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        # max over ranks
        m = bench.max_over_ranks(1.5 + rank, world)
        # replicas of the tables, distinct token batches
        w = bench.rank_workload(WORKLOADS["pkm"].scaled(T=16, H=2, d_half=32, n_sub=16, k=4,
                                                        d_v=16), rank)
        inp = make_inputs(w, "cpu")
        ksum = torch.tensor([float(inp["subkeys"].double().sum()),
                             float(inp["values"].double().sum())])
        qsum = torch.tensor([float(inp["query"].double().sum())])
        ks = [torch.zeros(2) for _ in range(world)]
        qs = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(ks, ksum)
        dist.all_gather(qs, qsum)
        # every rank runs its own units independently (here: the oracle)
        idx, _, _, _ = oracle.pkm_select(inp["query"], inp["subkeys"], w.k)
        dist.barrier()
        q.put((rank, m, [k.tolist() for k in ks], [x.item() for x in qs], idx.shape))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, ks, qs, shape in res:
        assert m == 2.5                       # max over ranks seen by every rank
        assert ks[0] == ks[1]                 # same tables on every rank
        assert qs[0] != qs[1]                 # distinct token batches
        assert shape == (16, 2, 4)


def test_whole_job_value():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.whole_job_tokens_per_s(8192, 1, 1.0) == 8192e3
    assert bench.whole_job_tokens_per_s(8192, 8, 2.0) == 8 * 8192 / 2e-3
    np.testing.assert_allclose(bench.whole_job_tokens_per_s(100, 3, 0.5), 600e3)


# ----------------------------------------------- launcher and sharded mode --

def _root():
    return os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_torchrun_command():
    import sys
    sys.path.insert(0, _root())
    import bench

    cmd = bench.torchrun_command(["--gpus", "4", "--steps", "3"], 4, 29512)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29512" in cmd
    assert cmd[-5].endswith("bench.py") and cmd[-4:] == ["--gpus", "4", "--steps", "3"]


def test_launcher_starts_two_ranks():
    """``bench.py --gpus 2`` run directly starts itself under
    torch.distributed.run; both ranks join one process group (gloo here, no
    GPU) and rank 0 prints the line."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(_root(), "bench.py"), "--gpus", "2",
                        "--launcher-check"], capture_output=True, text=True, timeout=300,
                       cwd=_root())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["rank_sum"] == 1.0


def test_launcher_rejects_world_mismatch():
    import subprocess
    import sys

    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(_root(), "bench.py"), "--gpus", "2",
                        "--launcher-check"], capture_output=True, text=True, timeout=300,
                       cwd=_root(), env=env)
    assert r.returncode != 0 and "--gpus 2 but 3 ranks" in r.stderr


def _select_ref(q, K, k):
    import oracle

    idx, _, w, _ = oracle.pkm_select(q, K, k)
    return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w).float()


def _gather_ref(shard, row_lo, idx, w):
    import oracle

    loc = idx.numpy().astype(np.int64) - row_lo
    mine = (loc >= 0) & (loc < shard.shape[0])
    return torch.from_numpy(oracle.bag(np.where(mine, loc, 0), np.where(mine, w.numpy(), 0.0),
                                       shard)).float()


def _sharded_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, _root())
    import argparse
    import datetime

    import bench
    from sparse_key_value_b200.inputs import WORKLOADS
    from sparse_key_value_b200.sharded import exchange_bytes, shard_rows

    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        w = WORKLOADS["pkm"].scaled(T=12, H=2, d_half=32, n_sub=16, k=4, d_v=16)
        args = argparse.Namespace(workload="pkm", workload_obj=w, steps=2, warmup=1)
        res = bench.run_sharded(args, rank, world, 0, select=_select_ref, gather=_gather_ref,
                                device="cpu")
        lo, n = shard_rows(w.N, world, rank)
        q.put((rank, res["n_gpus"], res["y_shape"], res["config"]["rows_per_rank"], n,
               res["exchange_bytes_per_rank"] == exchange_bytes(12, 2, 4, 16, world),
               res["value"] > 0, res["scaling"]))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_sharded_bench_step_two_ranks():
    """bench.py --sharded's step on two gloo ranks with the reference steps
    injected: each rank holds its share of the rows, the step order runs
    through the collectives and returns the rank's own bags."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, n_gpus, y_shape, rows, n_expect, xb_ok, positive, scaling in res:
        assert n_gpus == 2 and y_shape == [12, 16] and rows == n_expect == 128
        assert xb_ok and positive and scaling == "weak"
