"""GPU parity of the training backward against the CPU oracle (C ABI)."""

import numpy as np
import pytest
import torch

from parity import RTOL, close

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import WORKLOADS, make_inputs, random_bags  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    yield
    assert skv.device_error() == 0


def _oracle_selection(inp, k):
    import oracle
    idx, S, w, _ = oracle.pkm_select(inp["query"].cpu(), inp["subkeys"].cpu(), k)
    return idx, w


def run_backward(wl, dense=False, sample_rows=None):
    """GPU backward fed with the oracle's own selection and weights, against
    the oracle's backward on the same selection."""
    import oracle

    inp = make_inputs(wl, "cuda")
    idx_o, w_o = _oracle_selection(inp, wl.k)
    idx_g = torch.from_numpy(idx_o.astype(np.int32)).cuda()
    w_g = torch.from_numpy(w_o.astype(np.float32)).cuda()
    dense_t = torch.zeros(wl.N, wl.d_v, dtype=torch.float32, device="cuda") if dense else None
    g = skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx_g, w_g, inp["dy"],
                         dense=dense_t, want_dscores=True)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    rows = np.unique(idx_o)
    vrow = np.searchsorted(rows, idx_o)
    table = inp["values"][torch.from_numpy(rows).cuda()].cpu()
    ref = oracle.pkm_backward(inp["query"].cpu(), inp["subkeys"].cpu(), table, idx_o, vrow,
                              w_g.double().cpu().numpy(), inp["dy"].cpu(),
                              want_dv=sample_rows is None)
    rt = RTOL[wl.dtype]
    close(g["dscores"].cpu().numpy(), ref["dS"], rt, "dS")
    close(g["dquery"].cpu().numpy(), ref["dq"], rt, "dquery")
    close(g["dsubkeys"].cpu().numpy(), ref["dK"], rt, "dsubkeys")
    # sparse value gradient: exactly the selected rows, ascending
    got_rows = g["uniq_rows"].cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(got_rows, rows)
    assert int(g["n_uniq"].item()) == rows.shape[0]
    grad = g["grad_rows"].cpu().numpy()
    if sample_rows is None:
        close(grad, ref["dV"], rt, "grad_rows")
        if dense:
            close(dense_t[torch.from_numpy(rows).cuda()].cpu().numpy(), ref["dV"], rt, "dense")
            assert float(dense_t.abs().sum()) == pytest.approx(float(np.abs(grad).sum()), rel=1e-5)
    else:
        pick = np.unique(np.concatenate([rows[:3], rows[-3:],
                                         rows[np.linspace(0, len(rows) - 1, sample_rows)
                                              .astype(np.int64)]]))
        # the most popular rows too
        counts = np.bincount(np.searchsorted(rows, idx_o.ravel()), minlength=len(rows))
        pick = np.unique(np.concatenate([pick, rows[np.argsort(-counts)[:8]]]))
        ref_rows = oracle.value_grad_rows(idx_o, w_g.double().cpu().numpy(), inp["dy"].cpu(), pick)
        close(grad[np.searchsorted(rows, pick)], ref_rows, rt, "grad_rows (sampled)")
    return g, idx_o, rows


# bf16 with d_v a multiple of 256 (up to 2048) and at most a quarter as many
# slots as table rows takes the value-gradient walk that also yields dw (one
# warp per chunk of sorted entries and 512-column slice, rows through
# bulk-copy rings); other shapes re-gather the value rows for dw, and their
# bf16 rows of 1024..4096 columns (multiples of 512) are summed by the ring
# walk (one CTA per chunk, whole rows through bulk copies)
SMALL = [
    # name, T, H, d_half, n_sub, k, d_v, dtype, zipf
    ("bf16-small", 200, 2, 256, 64, 16, 128, "bf16", False),
    ("bf16-zipf", 300, 2, 256, 32, 32, 64, "bf16", True),
    ("bf16-dw-256", 64, 2, 256, 128, 8, 256, "bf16", False),
    ("bf16-dw-768-ragged", 70, 3, 256, 96, 7, 768, "bf16", False),
    ("bf16-dw-2048-zipf", 40, 2, 256, 128, 16, 2048, "bf16", True),
    ("bf16-redo-2048-zipf", 257, 2, 256, 64, 32, 2048, "bf16", True),
    # re-gathered dw, value rows of 1024..4096 columns summed by the ring walk
    ("bf16-ring-1024-zipf", 300, 2, 256, 64, 16, 1024, "bf16", True),
    ("bf16-ring-1536-ragged", 77, 3, 256, 40, 7, 1536, "bf16", False),
    ("bf16-ring-4096-zipf", 33, 1, 256, 32, 32, 4096, "bf16", True),
    ("f32-small", 130, 3, 128, 16, 8, 32, "f32", False),
    ("bf16-k1", 64, 1, 256, 8, 1, 16, "bf16", False),
    ("f32-k64", 50, 1, 128, 64, 64, 24, "f32", False),
    # wide query halves: the dq pass holds 16..64 query elements per lane
    ("bf16-dh1024", 40, 2, 1024, 32, 8, 64, "bf16", False),
    ("bf16-dh2048-k64", 24, 1, 2048, 64, 64, 32, "bf16", False),
    ("f32-dh512", 30, 2, 512, 32, 16, 48, "f32", False),
    ("f32-dh2048", 16, 1, 2048, 16, 8, 16, "f32", False),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_backward_small(case):
    name, T, H, dh, n, k, dv, dt, zipf = case
    base = WORKLOADS["train"]
    wl = base.scaled(name=name, T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv, dtype=dt,
                     seed=sum(map(ord, name)),
                     zipf_beta=base.zipf_beta if zipf else 0.0)
    run_backward(wl, dense=True)


def test_backward_deterministic():
    wl = WORKLOADS["train"].scaled(T=400, H=2, d_half=256, n_sub=32, k=32, d_v=256)
    inp = make_inputs(wl, "cuda")
    out, idx, w = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], wl.k)
    a = skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx, w, inp["dy"])
    b = skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx, w, inp["dy"])
    for key in ("dquery", "dsubkeys", "uniq_rows", "grad_rows"):
        assert torch.equal(a[key], b[key]), key


def test_backward_chained_after_forward():
    """GPU forward then GPU backward; where the selections agree the
    gradients match the oracle's."""
    import oracle

    wl = WORKLOADS["train"].scaled(T=128, H=2, d_half=256, n_sub=64, k=16, d_v=128, seed=77)
    inp = make_inputs(wl, "cuda")
    out, idx, w = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], wl.k)
    idx_o, w_o = _oracle_selection(inp, wl.k)
    if not np.array_equal(idx.cpu().numpy(), idx_o):
        pytest.skip("selection differs by a tie at this seed")
    g = skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx, w, inp["dy"])
    rows = np.unique(idx_o)
    ref = oracle.pkm_backward(inp["query"].cpu(), inp["subkeys"].cpu(),
                              inp["values"][torch.from_numpy(rows).cuda()].cpu(), idx_o,
                              np.searchsorted(rows, idx_o), w_o, inp["dy"].cpu())
    close(g["dquery"].cpu().numpy(), ref["dq"], 2e-2, "dquery")
    close(g["grad_rows"].cpu().numpy(), ref["dV"], 2e-2, "grad_rows")


def test_backward_train_workload_full_size():
    """The training workload (T=8192, N=2^20, Zipf-biased sub-keys): dq, dK,
    dS over all tokens, value-gradient rows sampled (hot rows included)."""
    wl = WORKLOADS["train"]
    g, idx_o, rows = run_backward(wl, sample_rows=48)
    counts = np.bincount(np.searchsorted(rows, idx_o.ravel()))
    print(f"train workload: {len(rows)} distinct rows of {idx_o.size} slots, "
          f"hottest row {counts.max()} contributions")


def test_backward_bad_row_id_sets_status():
    wl = WORKLOADS["train"].scaled(T=16, H=1, d_half=256, n_sub=8, k=4, d_v=16)
    inp = make_inputs(wl, "cuda")
    idx = torch.zeros(16, 1, 4, dtype=torch.int32, device="cuda")
    idx[:, 0, 1] = 1
    idx[:, 0, 2] = 2
    idx[:, 0, 3] = 3
    idx[5, 0, 2] = 64  # N = 64: out of range
    w = torch.full((16, 1, 4), 0.25, device="cuda")
    skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx, w, inp["dy"])
    assert skv.device_error() == 4


@pytest.mark.parametrize("n_bags,B,d,dt", [(100, 7, 24, "f32"), (300, 128, 256, "bf16"),
                                           (1, 1, 8, "bf16")])
def test_embbag_backward(n_bags, B, d, dt):
    import oracle

    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    n_rows = 500
    g = torch.Generator().manual_seed(B * 3 + d)
    table = (torch.randn(n_rows, d, generator=g) * 0.02).to(tdt).cuda()
    dy = torch.randn(n_bags, d, generator=g).to(tdt).cuda()
    idx, w = random_bags(n_bags, B, n_rows, seed=d, zipf=1.1)
    dense = torch.zeros(n_rows, d, device="cuda")
    res = skv.embbag_backward(dy, idx.cuda(), w.cuda(), table=table, dense=dense, want_dw=True)
    idx64 = idx.numpy().astype(np.int64).reshape(n_bags, 1, B)
    w64 = w.double().numpy().reshape(n_bags, 1, B)
    rows = np.unique(idx64)
    ref_rows = oracle.value_grad_rows(idx64, w64, dy.cpu(), rows)
    np.testing.assert_array_equal(res["uniq_rows"].cpu().numpy(), rows)
    close(res["grad_rows"].cpu().numpy(), ref_rows, RTOL[dt], "grad_rows")
    close(dense[torch.from_numpy(rows).cuda()].cpu().numpy(), ref_rows, RTOL[dt], "dense")
    # dw = <dy_t, table[idx]> (library einsum on the exact inputs, fp64)
    ref_dw = np.einsum("td,tbd->tb", dy.double().cpu().numpy(),
                       table.double().cpu().numpy()[idx.numpy()])
    close(res["dw"].cpu().numpy(), ref_dw, RTOL[dt], "dw")


# bf16 rows of 1024..4096 columns take the segmented sum whose source rows come
# through a ring of whole-row bulk copies (one CTA per chunk of sorted entries,
# a producer lane up to 12..32 rows ahead): hot rows span many chunks, the last
# chunk is ragged, 1536 columns puts three consumer warps on a row
@pytest.mark.parametrize("n_bags,B,d", [(700, 47, 1024), (130, 64, 1536), (90, 40, 4096)])
def test_embbag_backward_wide_rows(n_bags, B, d):
    import oracle

    n_rows = 3000
    g = torch.Generator().manual_seed(n_bags + d)
    dy = torch.randn(n_bags, d, generator=g).to(torch.bfloat16).cuda()
    idx, w = random_bags(n_bags, B, n_rows, seed=d + 1, zipf=1.1)
    dense = torch.zeros(n_rows, d, device="cuda")
    res = skv.embbag_backward(dy, idx.cuda(), w.cuda(), n_rows=n_rows, dense=dense)
    idx64 = idx.numpy().astype(np.int64).reshape(n_bags, 1, B)
    w64 = w.double().numpy().reshape(n_bags, 1, B)
    rows = np.unique(idx64)
    ref_rows = oracle.value_grad_rows(idx64, w64, dy.cpu(), rows)
    np.testing.assert_array_equal(res["uniq_rows"].cpu().numpy(), rows)
    close(res["grad_rows"].cpu().numpy(), ref_rows, RTOL["bf16"], "grad_rows")
    close(dense[torch.from_numpy(rows).cuda()].cpu().numpy(), ref_rows, RTOL["bf16"], "dense")
    # summed in sorted order: a second run gives the same bits
    res2 = skv.embbag_backward(dy, idx.cuda(), w.cuda(), n_rows=n_rows)
    assert torch.equal(res["grad_rows"], res2["grad_rows"])


def test_backward_side_stream_caller_stream_and_graph():
    """With dw from the per-slot re-gather, the value-gradient branch (sort and
    walk) runs on the library's second stream beside the rest of the
    backward and the caller's stream waits for it; inside a CUDA-graph
    capture it runs in line.  On a caller stream other than the default, and
    replayed from a graph, the results equal the eager ones bit for bit."""
    wl = WORKLOADS["train"].scaled(name="side-stream", T=300, H=2, d_half=256, n_sub=64, k=16,
                                   d_v=1024, seed=5)
    inp = make_inputs(wl, "cuda")
    q, K, V, dy = inp["query"], inp["subkeys"], inp["values"], inp["dy"]
    out, idx, w = skv.pkm_forward(q, K, V, wl.k)
    N = wl.n_sub ** 2
    assert wl.T * wl.H * wl.k * 4 > N  # the re-gather path, where the branches split

    def run(dense):
        return skv.pkm_backward(q, K, V, idx, w, dy, sparse=False, dense=dense)

    d0 = torch.zeros(N, wl.d_v, device="cuda")
    a = run(d0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    d1 = torch.zeros(N, wl.d_v, device="cuda")
    with torch.cuda.stream(s):
        b = run(d1)
    s.synchronize()
    d2 = torch.zeros(N, wl.d_v, device="cuda")
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(torch.zeros(N, wl.d_v, device="cuda"))  # warm the allocator outside the capture
    side.synchronize()
    with torch.cuda.graph(g):
        c = run(d2)
    d2.zero_()
    g.replay()
    torch.cuda.synchronize()
    for key in ("dquery", "dsubkeys"):
        assert torch.equal(a[key], b[key]), key
        assert torch.equal(a[key], c[key]), key
    assert torch.equal(d0, d1)
    assert torch.equal(d0, d2)
    assert skv.device_error() == 0


def test_embbag_backward_wide_rows_invalid_ids():
    """Out-of-range row ids (negative or past the table) in the ring walk's
    value gradient: those entries are dropped (sorted last, never summed), the
    device status records the anomaly, and every valid row's gradient is
    exact against the oracle on the valid entries alone."""
    import oracle

    n_bags, B, d, n_rows = 500, 40, 1024, 2000
    g = torch.Generator().manual_seed(77)
    dy = torch.randn(n_bags, d, generator=g).to(torch.bfloat16).cuda()
    idx, w = random_bags(n_bags, B, n_rows, seed=78, zipf=1.1)
    bad = torch.rand(n_bags, B, generator=g) < 0.01
    idx[bad & (torch.rand(n_bags, B, generator=g) < 0.5)] = -1
    idx[bad & (idx >= 0)] = n_rows + 5
    assert int(bad.sum()) > 0
    res = skv.embbag_backward(dy, idx.cuda(), w.cuda(), n_rows=n_rows)
    assert skv.device_error() == 4  # PKM_ERR_DEVICE: an out-of-range row id
    idx64 = idx.numpy().astype(np.int64)
    valid = (idx64 >= 0) & (idx64 < n_rows)
    rows = np.unique(idx64[valid])
    # the invalid entries contribute nothing: weight 0 on a row that is present anyway
    idx_ok = np.where(valid, idx64, rows[0]).reshape(n_bags, 1, B)
    w_ok = np.where(valid, w.double().numpy(), 0.0).reshape(n_bags, 1, B)
    ref_rows = oracle.value_grad_rows(idx_ok, w_ok, dy.cpu(), rows)
    np.testing.assert_array_equal(res["uniq_rows"].cpu().numpy(), rows)
    close(res["grad_rows"].cpu().numpy(), ref_rows, RTOL["bf16"], "grad_rows")
