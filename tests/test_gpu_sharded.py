"""GPU parity of the row-sharded lookup's two CUDA steps, through the C ABI:
pkm_select (the selection alone) and embbag_forward_range (one shard's fp32
partial bags).  One GPU holds every shard here: the shards' partials, summed
in shard order, must give the oracle's bag over the whole table, which is
what the reduce-scatter of sparse_key_value_b200.sharded computes across
ranks (that exchange is tested on the host with gloo ranks)."""

import numpy as np
import pytest
import torch

from parity import RTOL, close

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import WORKLOADS, make_inputs  # noqa: E402
from sparse_key_value_b200.sharded import shard_rows, sharded_lookup  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    yield
    assert skv.device_error() == 0


CASES = [("tc", 300, 2, 128, 512, 16, 256, "bf16"), ("simt-f32", 90, 2, 32, 64, 8, 40, "f32")]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_select_equals_the_forwards_selection(case):
    name, T, H, dh, n, k, dv, dt = case
    w = WORKLOADS["pkm"].scaled(T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv, dtype=dt, seed=5)
    inp = make_inputs(w, "cuda")
    _, idx_f, w_f = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], k)
    idx_s, w_s = skv.pkm_select(inp["query"], inp["subkeys"], k, d_v=dv)
    torch.cuda.synchronize()
    assert torch.equal(idx_f, idx_s) and torch.equal(w_f, w_s)


def _partials(values, idx2, w2, G):
    N = values.shape[0]
    total = None
    for r in range(G):
        lo, n = shard_rows(N, G, r)
        if n == 0:
            continue
        p = skv.embbag_forward_range(values[lo:lo + n], lo, idx2, w2)
        total = p if total is None else total + p  # shard order
    return total


@pytest.mark.parametrize("G", [1, 2, 3, 8])
def test_shard_partials_sum_to_the_full_bag(G):
    import oracle

    w = WORKLOADS["pkm"].scaled(T=200, H=2, d_half=128, n_sub=256, k=16, d_v=512, seed=6)
    inp = make_inputs(w, "cuda")
    idx, wt = skv.pkm_select(inp["query"], inp["subkeys"], w.k, d_v=w.d_v)
    idx2, w2 = idx.view(w.T, -1), wt.view(w.T, -1)
    y = _partials(inp["values"], idx2, w2, G)
    torch.cuda.synchronize()
    assert skv.device_error() == 0  # ids of other shards are not an error
    ids = idx2.cpu().numpy().astype(np.int64)
    rows = np.unique(ids)
    table = inp["values"][torch.from_numpy(rows).cuda()].cpu()
    ref = oracle.bag(np.searchsorted(rows, ids), w2.double().cpu().numpy(), table)
    close(y.double().cpu().numpy(), ref, RTOL["f32"], f"sum of {G} shards")


def test_sharded_lookup_one_rank():
    """sparse_key_value_b200.sharded.sharded_lookup with its CUDA defaults on
    one rank (the collectives are the identity)."""
    import oracle

    class One:
        def all_gather(self, t):
            return t.unsqueeze(0)

        def reduce_scatter_sum(self, t):
            return t

    w = WORKLOADS["pkm"].scaled(T=64 + 37, H=2, d_half=64, n_sub=256, k=8, d_v=256, seed=7)
    inp = make_inputs(w, "cuda")
    y, idx, wt = sharded_lookup(inp["query"], inp["subkeys"], inp["values"], w.k, 0, One())
    torch.cuda.synchronize()
    ids = idx.view(w.T, -1).cpu().numpy().astype(np.int64)
    rows = np.unique(ids)
    table = inp["values"][torch.from_numpy(rows).cuda()].cpu()
    ref = oracle.bag(np.searchsorted(rows, ids), wt.view(w.T, -1).double().cpu().numpy(), table)
    close(y.double().cpu().numpy(), ref, RTOL["f32"], "sharded lookup, one rank")


def test_range_ids_outside_every_shard_row():
    """A bag whose ids all lie in other shards is exactly zero."""
    values = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    idx = torch.tensor([[0, 1, 2], [50, 60, 99]], dtype=torch.int32, device="cuda")
    w = torch.ones(2, 3, device="cuda")
    out = skv.embbag_forward_range(values[50:], 50, idx, w)
    torch.cuda.synchronize()
    assert torch.equal(out[0], torch.zeros(64, device="cuda"))
    ref = values[50].float() + values[60].float() + values[99].float()
    torch.testing.assert_close(out[1], ref, rtol=1e-6, atol=1e-6)


def test_pkm_workload_over_eight_shards_sampled():
    """The PKM workload (T = 8192, 2^20 x 2048 table) over eight row shards
    held on one GPU: sampled tokens against the oracle."""
    import oracle

    w = WORKLOADS["pkm"]
    inp = make_inputs(w, "cuda")
    idx, wt = skv.pkm_select(inp["query"], inp["subkeys"], w.k, d_v=w.d_v)
    idx2, w2 = idx.view(w.T, -1), wt.view(w.T, -1)
    y = _partials(inp["values"], idx2, w2, 8)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(8)
    sample = torch.cat([torch.tensor([0, w.T - 1]), torch.randperm(w.T, generator=g)[:62]])
    ids = idx2[sample.cuda()].cpu().numpy().astype(np.int64)
    rows = np.unique(ids)
    table = inp["values"][torch.from_numpy(rows).cuda()].cpu()
    ref = oracle.bag(np.searchsorted(rows, ids), w2[sample.cuda()].double().cpu().numpy(), table)
    close(y[sample.cuda()].double().cpu().numpy(), ref, RTOL["f32"], "eight shards")
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,d,dt", [(70, 256, "bf16"), (1, 64, "bf16"), (33, 128, "f32"),
                                    (300, 1024, "bf16")])
def test_range_gather_odd_bags_against_oracle(B, d, dt):
    """Bags whose size is not a multiple of the 32-entry compaction step,
    single-entry bags and fp32 tables, over three uneven shards."""
    import oracle
    from sparse_key_value_b200.inputs import random_bags

    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    n_rows, n_bags = 1001, 45
    g = torch.Generator().manual_seed(B + d)
    table = (torch.randn(n_rows, d, generator=g) * 0.02).to(tdt).cuda()
    idx, w = random_bags(n_bags, B, n_rows, seed=B * 7 + d)
    idx, w = idx.cuda(), w.cuda()
    cuts = [0, 13, 600, n_rows]  # uneven shares
    y = None
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        p = skv.embbag_forward_range(table[lo:hi], lo, idx, w)
        y = p if y is None else y + p
    torch.cuda.synchronize()
    ref = oracle.bag(idx.cpu().numpy().astype(np.int64), w.double().cpu().numpy(), table.cpu())
    close(y.double().cpu().numpy(), ref, RTOL["f32"], f"B={B} d={d} {dt}")
