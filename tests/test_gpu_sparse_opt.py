"""GPU parity of the optimiser step on the touched value rows ("모델 안의
메모리", "잊지 않고 배우기": only the slots a fact uses are updated) against
the CPU oracle, through the C ABI."""

import numpy as np
import pytest
import torch

from parity import RTOL, close

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    yield
    assert skv.device_error() == 0


def _case(seed, n_rows=500, d=64, n=37, cap=48):
    g = torch.Generator().manual_seed(seed)
    table = torch.randn(n_rows, d, generator=g) * 0.02
    rows = torch.randperm(n_rows, generator=g)[:cap].to(torch.int32)
    grads = torch.randn(cap, d, generator=g)
    count = torch.tensor([n], dtype=torch.int64)
    return table, rows, grads, count


def test_sgd_fp32_matches_oracle():
    import oracle

    table, rows, grads, count = _case(1)
    t = table.cuda()
    skv.sparse_optimizer_step(t, rows.cuda(), grads.cuda(), count.cuda(), lr=0.05)
    torch.cuda.synchronize()
    n = int(count)
    ref = oracle.sparse_sgd(table.double().numpy(), rows[:n].numpy(), grads[:n].double().numpy(),
                            0.05)
    np.testing.assert_allclose(t.cpu().double().numpy(), ref, rtol=1e-6, atol=1e-8)
    # entries past the count are not applied
    untouched = np.setdiff1d(np.arange(table.shape[0]), rows[:n].numpy())
    assert torch.equal(t.cpu()[untouched], table[untouched])


def test_adam_fp32_three_steps_match_oracle():
    import oracle

    table, _, _, _ = _case(2)
    t = table.cuda()
    m = torch.zeros_like(t)
    v = torch.zeros_like(t)
    rt, rm, rv = table.double().numpy(), np.zeros(table.shape), np.zeros(table.shape)
    for step in (1, 2, 3):
        _, rows, grads, count = _case(10 + step)
        skv.sparse_optimizer_step(t, rows.cuda(), grads.cuda(), count.cuda(), lr=0.01,
                                  kind="adam", m=m, v=v, betas=(0.9, 0.99), eps=1e-6, step=step)
        n = int(count)
        rt, rm, rv = oracle.sparse_adam(rt, rm, rv, rows[:n].numpy(), grads[:n].double().numpy(),
                                        0.01, 0.9, 0.99, 1e-6, step)
    torch.cuda.synchronize()
    np.testing.assert_allclose(t.cpu().double().numpy(), rt, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(m.cpu().double().numpy(), rm, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(v.cpu().double().numpy(), rv, rtol=1e-5, atol=1e-7)


def test_sgd_bf16_rounds_once():
    """bf16 table: the fp32 update rounded once to nearest even equals the
    oracle's update rounded the same way (up to one ulp where fp32 and fp64
    straddle a rounding boundary)."""
    import oracle

    table, rows, grads, count = _case(3)
    tb = table.to(torch.bfloat16)
    t = tb.cuda()
    skv.sparse_optimizer_step(t, rows.cuda(), grads.cuda(), count.cuda(), lr=0.5)
    torch.cuda.synchronize()
    n = int(count)
    ref = oracle.sparse_sgd(tb.double().numpy(), rows[:n].numpy(), grads[:n].double().numpy(),
                            0.5)
    ref_b = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int32)
    got = t.cpu().view(torch.int16).numpy().astype(np.int32)
    assert np.max(np.abs(got - ref_b)) <= 1


def test_step_on_backward_output():
    """The backward's sparse value gradient drives the step: exactly the
    selected rows change, by lr times their gradient rows."""
    w = WORKLOADS["train"].scaled(T=200, H=2, d_half=256, n_sub=64, k=8, d_v=64)
    inp = make_inputs(w, "cuda")
    out, idx, wts = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    g = skv.pkm_backward(inp["query"], inp["subkeys"], inp["values"], idx, wts, inp["dy"])
    table = inp["values"].float().clone()
    before = table.clone()
    skv.sparse_optimizer_step(table, g["uniq_rows"], g["grad_rows"], g["n_uniq"], lr=0.1)
    torch.cuda.synchronize()
    n = int(g["n_uniq"].item())
    rows = g["uniq_rows"][:n].long()
    assert torch.equal(torch.unique(idx.long()), rows)
    torch.testing.assert_close(table[rows], before[rows] - 0.1 * g["grad_rows"][:n],
                               rtol=1e-6, atol=1e-7)
    mask = torch.ones(table.shape[0], dtype=torch.bool, device="cuda")
    mask[rows] = False
    assert torch.equal(table[mask], before[mask])


def test_shared_pool_gradient_in_one_reduction():
    """"Memory Layers at Scale" digest, "공유 메모리 풀": several layers read one
    value pool.  Each layer's forward writes its selection into its slice of
    one layer-major buffer; the pool's sparse value gradient is then one
    sorted segmented sum over all layers' slots (embbag_backward), equal to
    the oracle's sum over the layers and to per-layer gradients added
    densely."""
    import oracle

    L = 3
    w = WORKLOADS["train"].scaled(T=128, H=2, d_half=256, n_sub=64, k=8, d_v=64)
    pool = make_inputs(w, "cuda")["values"]
    T, B = w.T, w.H * w.k
    idx = torch.empty(L * T, B, dtype=torch.int32, device="cuda")
    wts = torch.empty(L * T, B, dtype=torch.float32, device="cuda")
    g = torch.Generator().manual_seed(41)
    dy = torch.randn(L * T, w.d_v, generator=g).to(torch.bfloat16).cuda()
    for layer in range(L):
        lw = w.scaled(seed=w.seed + 100 * (layer + 1), table_seed_=w.seed + 200 * (layer + 1))
        li = make_inputs(lw, "cuda", with_values=False)
        s = slice(layer * T, (layer + 1) * T)
        skv.pkm_forward(li["query"], li["subkeys"], pool, w.k, idx=idx[s].view(T, w.H, w.k),
                        weights=wts[s].view(T, w.H, w.k))
    res = skv.embbag_backward(dy, idx, wts, n_rows=pool.shape[0])
    dense = torch.zeros(pool.shape[0], w.d_v, dtype=torch.float32, device="cuda")
    for layer in range(L):
        s = slice(layer * T, (layer + 1) * T)
        skv.embbag_backward(dy[s], idx[s], wts[s], n_rows=pool.shape[0], sparse=False,
                            dense=dense)
    torch.cuda.synchronize()
    rows = np.unique(idx.cpu().numpy().astype(np.int64))
    np.testing.assert_array_equal(res["uniq_rows"].cpu().numpy(), rows)
    ref = oracle.value_grad_rows(idx.cpu().numpy().astype(np.int64).reshape(L * T, 1, B),
                                 wts.double().cpu().numpy().reshape(L * T, 1, B), dy.cpu(), rows)
    close(res["grad_rows"].cpu().numpy(), ref, RTOL["f32"], "pool grad_rows")
    close(dense[torch.from_numpy(rows).cuda()].cpu().numpy(), ref, RTOL["f32"],
          "per-layer dense sum")
