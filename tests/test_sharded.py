"""The row-sharded lookup's exchange logic on the host: two and three gloo
ranks (no GPU), each holding a contiguous share of the value table.

The selection and the partial gather are the oracle here (fp64, injected
into sparse_key_value_b200.sharded.sharded_lookup); on a GPU the same
function calls the CUDA library's pkm_select and embbag_forward_range
(tests/test_gpu_sharded.py).  What is checked is the exchange: the
all-gather of the selections, every rank summing the rows it holds for all
ranks' tokens, and the reduce-scatter handing each rank the full bags of its
own tokens -- equal to the oracle's bag over the whole table.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_select(q, K, k):
    import oracle

    idx, _, w, _ = oracle.pkm_select(q, K, k)
    return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)


def _oracle_range_gather(shard, row_lo, idx, w):
    """fp64 partial bags: rows outside [row_lo, row_lo + len(shard)) skipped."""
    import oracle

    loc = idx.numpy().astype(np.int64) - row_lo
    mine = (loc >= 0) & (loc < shard.shape[0])
    return torch.from_numpy(oracle.bag(np.where(mine, loc, 0), np.where(mine, w.numpy(), 0.0),
                                       shard))


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import datetime

    import oracle
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs
    from sparse_key_value_b200.sharded import TorchComm, shard_rows, sharded_lookup

    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=60))
        base = WORKLOADS["pkm"].scaled(T=12, H=2, d_half=32, n_sub=8, k=4, d_v=16, dtype="f32")
        w = base.scaled(seed=base.seed + 101 * rank, table_seed_=base.seed)
        inp = make_inputs(w, "cpu")  # own tokens, the same tables on every rank
        V = inp["values"].double()
        lo, n = shard_rows(w.N, world, rank)
        y, idx, wt = sharded_lookup(inp["query"], inp["subkeys"], V[lo:lo + n], w.k, lo,
                                    TorchComm(), select=_oracle_select,
                                    gather=_oracle_range_gather)
        ref = oracle.bag(idx.numpy().astype(np.int64).reshape(w.T, -1),
                         wt.numpy().reshape(w.T, -1), V)
        q.put((rank, float(np.abs(y.numpy() - ref).max()), float(np.abs(ref).max()), lo, n))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_row_sharded_lookup_equals_full_table(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in res] == list(range(world))
    assert sum(r[4] for r in res) == 64  # the shares cover the 8 x 8 rows exactly once
    for rank, err, mag, lo, n in res:
        assert mag > 0
        assert err <= 1e-12 * mag, (rank, err)


def test_shard_rows_cover_the_table_once():
    from sparse_key_value_b200.sharded import shard_rows

    for n_rows in (1, 7, 64, 1 << 20, (1 << 20) + 3):
        for world in (1, 2, 3, 8):
            shares = [shard_rows(n_rows, world, r) for r in range(world)]
            covered = np.zeros(n_rows, dtype=np.int64) if n_rows < 100 else None
            pos = 0
            for lo, n in shares:
                assert lo == pos and n >= 0
                pos += n
                if covered is not None:
                    covered[lo:lo + n] += 1
            assert pos == n_rows
            if covered is not None:
                assert np.all(covered == 1)
