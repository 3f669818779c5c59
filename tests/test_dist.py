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
