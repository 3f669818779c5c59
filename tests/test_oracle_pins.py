"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test ties one oracle function to brute force, a closed form, an
invariant, a library routine on a special case, the pages' printed counts,
or finite differences.  A plausible slip in the oracle (a wrong scale, a
swapped half, a transposed weight, a dropped softmax term, a wrong sign in
the backward) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from sparse_key_value_b200.inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * std).numpy()


def _problem(T, H, dh, n, seed):
    q = _rand((T, H, 2, dh), seed)
    K = _rand((H, 2, n, dh), seed + 1, 1.0 / math.sqrt(dh))
    return q, K


# --------------------------------------------------------------------------
# half scores: closed forms, invariance, library special case
# --------------------------------------------------------------------------

def test_half_scores_closed_forms(orc):
    dh, n = 16, 5
    q = _rand((1, 1, 2, dh), 3)
    K = _rand((1, 2, n, dh), 4)
    K[0, 0, 1] = 3.0 * q[0, 0, 0]       # parallel to the first half -> +sqrt(dh)
    K[0, 0, 2] = -0.5 * q[0, 0, 0]      # anti-parallel -> -sqrt(dh)
    v = _rand((dh,), 5)
    u = q[0, 0, 1]
    K[0, 1, 3] = v - (v @ u) / (u @ u) * u  # orthogonal to the second half -> 0
    s = orc.half_scores(q, K)
    assert s.shape == (1, 1, 2, n)
    assert s[0, 0, 0, 1] == pytest.approx(math.sqrt(dh), rel=1e-13)
    assert s[0, 0, 0, 2] == pytest.approx(-math.sqrt(dh), rel=1e-13)
    assert abs(s[0, 0, 1, 3]) < 1e-12
    assert np.all(np.abs(s) <= math.sqrt(dh) * (1 + 1e-12))


def test_half_scores_scale_invariance(orc):
    q, K = _problem(6, 2, 8, 7, 10)
    s = orc.half_scores(q, K)
    rng = np.random.default_rng(0)
    q2 = q * rng.uniform(0.01, 100.0, size=q.shape[:-1] + (1,))
    K2 = K * rng.uniform(0.01, 100.0, size=K.shape[:-1] + (1,))
    np.testing.assert_allclose(orc.half_scores(q2, K2), s, rtol=1e-12, atol=1e-12)


def test_half_scores_match_library_cosine(orc):
    q, K = _problem(4, 3, 12, 9, 11)
    s = orc.half_scores(q, K)
    qt, Kt = torch.from_numpy(q), torch.from_numpy(K)
    for h in range(3):
        for c in range(2):
            cos = torch.nn.functional.cosine_similarity(
                qt[:, h, c, None, :], Kt[None, h, c, :, :], dim=-1)
            np.testing.assert_allclose(s[:, h, c, :], math.sqrt(12) * cos.numpy(),
                                       rtol=1e-12, atol=1e-12)


def test_zero_vector_clamp(orc):
    q = np.zeros((1, 1, 2, 4))
    K = _rand((1, 2, 3, 4), 12)
    assert np.all(orc.half_scores(q, K) == 0.0)


# --------------------------------------------------------------------------
# top-k and the tie rule: library sort
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (64, 64), (100, 17)])
def test_topk_matches_library_lexsort(orc, n, k):
    rng = np.random.default_rng(n * 100 + k)
    s = np.round(rng.normal(size=n), 1)  # many exact ties
    ref = np.lexsort((np.arange(n), -s))[:k]
    np.testing.assert_array_equal(orc.topk(s, k), ref)


def test_topk_matches_torch_on_distinct(orc):
    rng = np.random.default_rng(1)
    s = rng.normal(size=257)
    ref = torch.topk(torch.from_numpy(s), 31, sorted=True).indices.numpy()
    np.testing.assert_array_equal(orc.topk(s, 31), ref)


# --------------------------------------------------------------------------
# product-key selection == the definition (brute force over all N keys)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [2, 3, 8, 16])
def test_product_key_equals_bruteforce(orc, n):
    for k in sorted({1, 2, n // 2 or 1, n}):
        q, K = _problem(9, 2, 8, n, 20 + n * 10 + k)
        idx, S, w, _ = orc.pkm_select(q, K, k)
        bidx, bS = orc.bruteforce_select(q, K, k)
        np.testing.assert_array_equal(idx, bidx)
        np.testing.assert_allclose(S, bS, rtol=0, atol=1e-12)


def test_product_key_equals_bruteforce_tiny_workload(orc):
    """The tiny fp32 workload (N = 1024 keys): the definition brute-forced."""
    w = WORKLOADS["tiny"]
    inp = make_inputs(w.scaled(T=64), "cpu", with_values=False)
    idx, S, _, _ = orc.pkm_select(inp["query"], inp["subkeys"], w.k)
    bidx, bS = orc.bruteforce_select(inp["query"], inp["subkeys"], w.k)
    np.testing.assert_array_equal(idx, bidx)
    np.testing.assert_allclose(S, bS, rtol=0, atol=1e-12)


def test_selection_with_exact_ties(orc):
    """Duplicate sub-key rows tie exactly; the smaller row id comes first."""
    q, K = _problem(5, 1, 8, 6, 30)
    K[0, 0, 4] = K[0, 0, 1]
    K[0, 1, 5] = K[0, 1, 2]
    for k in (1, 3, 6):
        idx, _, _, _ = orc.pkm_select(q, K, k)
        bidx, _ = orc.bruteforce_select(q, K, k)
        np.testing.assert_array_equal(idx, bidx)


def test_planted_key_row_id_convention(orc):
    """Sub-key a* of half 1 equal to the first query half and b* of half 2
    equal to the second give the best full key, row id a* * n + b*."""
    n, dh = 11, 8
    q, K = _problem(3, 2, dh, n, 40)
    plants = {(0, 0): (7, 2), (0, 1): (3, 9), (1, 0): (10, 0), (2, 1): (0, 10)}
    for (t, h), (a, b) in plants.items():
        Kp = K.copy()
        Kp[h, 0, a] = 2.0 * q[t, h, 0]
        Kp[h, 1, b] = 5.0 * q[t, h, 1]
        idx, S, _, _ = orc.pkm_select(q, Kp, 1)
        assert idx[t, h, 0] == a * n + b
        assert S[t, h, 0] == pytest.approx(2 * math.sqrt(dh), rel=1e-12)


def test_k1_is_argmax_of_each_half(orc):
    q, K = _problem(7, 3, 8, 13, 50)
    s = orc.half_scores(q, K)
    idx, _, w, _ = orc.pkm_select(q, K, 1)
    np.testing.assert_array_equal(idx[..., 0], s[:, :, 0].argmax(-1) * 13 + s[:, :, 1].argmax(-1))
    assert np.all(w == 1.0)


def test_comparison_counts_match_pages(orc):
    """2*sqrt(N) half-key comparisons per (token, head), as the pages count."""
    with open(os.path.join(GOLDEN, "comparison_counts.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        n = case["n_sub"]
        assert n * n == case["cells"]
        q, K = _problem(2, 1, 4, n, 60)
        _, _, _, dots = orc.pkm_select(q, K, 2)
        assert dots == 2 * case["comparisons"]  # 2 (token, head) pairs
        assert dots // 2 == 2 * math.isqrt(case["cells"])


# --------------------------------------------------------------------------
# softmax weights
# --------------------------------------------------------------------------

def test_softmax_properties(orc):
    q, K = _problem(8, 2, 8, 10, 70)
    idx, S, w, _ = orc.pkm_select(q, K, 6)
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-14)
    ref = torch.softmax(torch.from_numpy(S), dim=-1).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-14, atol=0)
    assert np.all(np.diff(w, axis=-1) <= 0)  # scores are in descending order
    np.testing.assert_allclose(orc.softmax(np.full((3, 5), 2.5)), 0.2, rtol=1e-15)


# --------------------------------------------------------------------------
# weighted bag: library embedding_bag
# --------------------------------------------------------------------------

def test_bag_matches_library_embedding_bag(orc):
    rng = np.random.default_rng(2)
    table = rng.normal(size=(50, 24))
    idx = rng.integers(0, 50, size=(13, 9))
    w = rng.uniform(size=(13, 9))
    y = orc.bag(idx, w, table)
    ref = torch.nn.functional.embedding_bag(
        torch.from_numpy(idx), torch.from_numpy(table), mode="sum",
        per_sample_weights=torch.from_numpy(w)).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)


def test_bag_equal_scores_is_mean(orc):
    """Equal scores give w = 1/k: the bag is the plain mean of the rows."""
    rng = np.random.default_rng(3)
    table = rng.normal(size=(20, 8))
    idx = rng.integers(0, 20, size=(4, 5))
    w = orc.softmax(np.zeros((4, 5)))
    np.testing.assert_allclose(orc.bag(idx, w, table), table[idx].mean(1), rtol=1e-13)


def test_bag_bf16_decoding_exact(orc):
    t = torch.randn(9, 16, dtype=torch.float32).to(torch.bfloat16)
    idx = np.arange(9).reshape(9, 1)
    y = orc.bag(idx, np.ones((9, 1)), t)
    np.testing.assert_array_equal(y, t.double().numpy())


# --------------------------------------------------------------------------
# Memory+ gate: closed forms and library special cases
# --------------------------------------------------------------------------

def test_memplus_zero_gate(orc):
    rng = np.random.default_rng(4)
    y, x = rng.normal(size=(5, 6)), rng.normal(size=(5, 4))
    out = orc.memplus(y, x, np.zeros((4, 6)), rng.normal(size=(6, 4)))
    assert np.all(out == 0.0)


def test_memplus_identity_projection(orc):
    """W2 = I and y = 1: out = silu(x W1) (library silu and matmul)."""
    rng = np.random.default_rng(5)
    x, W1 = rng.normal(size=(7, 6)), rng.normal(size=(6, 6))
    out = orc.memplus(np.ones((7, 6)), x, W1, np.eye(6))
    ref = torch.nn.functional.silu(torch.from_numpy(x) @ torch.from_numpy(W1)).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_memplus_identity_gate_weights(orc):
    """W1 = I (d_model = d_v), y random: out = (y ⊙ silu(x)) W2 with a
    non-symmetric W2 (a transposed W2 fails)."""
    rng = np.random.default_rng(6)
    y, x, W2 = rng.normal(size=(4, 5)), rng.normal(size=(4, 5)), rng.normal(size=(5, 5))
    out = orc.memplus(y, x, np.eye(5), W2)
    g = torch.nn.functional.silu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(out, (y * g) @ W2, rtol=1e-13, atol=1e-15)
    assert not np.allclose(out, (y * g) @ W2.T)


def test_memplus_rectangular_shapes(orc):
    rng = np.random.default_rng(7)
    y, x = rng.normal(size=(3, 5)), rng.normal(size=(3, 2))
    W1, W2 = rng.normal(size=(2, 5)), rng.normal(size=(5, 2))
    out = orc.memplus(y, x, W1, W2)
    assert out.shape == (3, 2)
    # linear in y
    np.testing.assert_allclose(orc.memplus(2.5 * y, x, W1, W2), 2.5 * out, rtol=1e-13)


# --------------------------------------------------------------------------
# backward: central finite differences with the selection held fixed
# --------------------------------------------------------------------------

def _forward_fixed(orc, q, K, V, idx, n):
    """y from the oracle's own pieces with a fixed selection idx [T,H,k]."""
    s = orc.half_scores(q, K)  # [T,H,2,n]
    a, b = idx // n, idx % n
    T, H, k = idx.shape
    S = np.take_along_axis(s[:, :, 0], a, -1) + np.take_along_axis(s[:, :, 1], b, -1)
    w = orc.softmax(S)
    return orc.bag(idx.reshape(T, H * k), w.reshape(T, H * k), V)


def test_backward_finite_differences(orc):
    T, H, dh, n, k, dv = 3, 2, 4, 5, 3, 6
    q, K = _problem(T, H, dh, n, 80)
    V = _rand((n * n, dv), 81)
    dy = _rand((T, dv), 82)
    idx, S, w, _ = orc.pkm_select(q, K, k)
    g = orc.pkm_backward(q, K, V, idx, idx, w, dy)

    def loss(q_, K_, V_):
        return float(np.sum(dy * _forward_fixed(orc, q_, K_, V_, idx, n)))

    eps = 1e-6
    for name, arr, grad in (("q", q, g["dq"]), ("K", K, g["dK"]), ("V", V, g["dV"])):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            p, m = arr.copy(), arr.copy()
            p[i] += eps
            m[i] -= eps
            args = {"q": (q, K, V), "K": (q, K, V), "V": (q, K, V)}[name]
            ap = [p if nm == name else a for nm, a in zip("qKV", args)]
            am = [m if nm == name else a for nm, a in zip("qKV", args)]
            num[i] = (loss(*ap) - loss(*am)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)

    # dw = <dy_t, V[idx]>; dS sums to zero per (t, h) (softmax Jacobian)
    np.testing.assert_allclose(g["dS"].sum(-1), 0.0, atol=1e-14)
    np.testing.assert_allclose(g["dw"], np.einsum("td,thkd->thk", dy, V[idx]), rtol=1e-13)


def test_backward_matches_autograd(orc):
    """torch.autograd (CPU, fp64) on the same composition, as a second check."""
    T, H, dh, n, k, dv = 4, 2, 6, 4, 3, 3
    q, K = _problem(T, H, dh, n, 90)
    V = _rand((n * n, dv), 91)
    dy = _rand((T, dv), 92)
    idx, _, w, _ = orc.pkm_select(q, K, k)
    g = orc.pkm_backward(q, K, V, idx, idx, w, dy)
    qt = torch.tensor(q, requires_grad=True)
    Kt = torch.tensor(K, requires_grad=True)
    Vt = torch.tensor(V, requires_grad=True)
    u = qt / qt.norm(dim=-1, keepdim=True)
    kap = Kt / Kt.norm(dim=-1, keepdim=True)
    s = math.sqrt(dh) * torch.einsum("thcd,hcnd->thcn", u, kap)
    it = torch.from_numpy(idx)
    S = torch.gather(s[:, :, 0], -1, it // n) + torch.gather(s[:, :, 1], -1, it % n)
    y = (torch.softmax(S, -1).unsqueeze(-1) * Vt[it]).sum((1, 2))
    (y * torch.from_numpy(dy)).sum().backward()
    np.testing.assert_allclose(g["dq"], qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dK"], Kt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dV"], Vt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_compact_rows(orc):
    """dV accumulated on a compact table equals the full-table result."""
    T, H, dh, n, k, dv = 5, 2, 4, 6, 4, 3
    q, K = _problem(T, H, dh, n, 95)
    V = _rand((n * n, dv), 96)
    dy = _rand((T, dv), 97)
    idx, _, w, _ = orc.pkm_select(q, K, k)
    full = orc.pkm_backward(q, K, V, idx, idx, w, dy)
    uniq, inv = np.unique(idx, return_inverse=True)
    comp = orc.pkm_backward(q, K, V[uniq], idx, inv.reshape(idx.shape), w, dy)
    np.testing.assert_allclose(comp["dV"], full["dV"][uniq], rtol=1e-13)
    np.testing.assert_array_equal(comp["dq"], full["dq"])


def test_value_grad_rows_matches_backward(orc):
    """The row-sampled value gradient equals the (finite-difference pinned)
    full backward's dV on the same rows."""
    T, H, dh, n, k, dv = 6, 2, 4, 5, 3, 7
    q, K = _problem(T, H, dh, n, 98)
    V = _rand((n * n, dv), 99)
    dy = _rand((T, dv), 100)
    idx, _, w, _ = orc.pkm_select(q, K, k)
    full = orc.pkm_backward(q, K, V, idx, idx, w, dy)
    rows = np.array(sorted(set(idx.ravel().tolist()))[::2] + [n * n - 1])
    got = orc.value_grad_rows(idx, w, dy, rows)
    np.testing.assert_allclose(got, full["dV"][rows], rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# Memory+ backward and the query projection
# --------------------------------------------------------------------------

def _memplus_inputs(seed, T=6, dm=5, dv=7):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(T, dv)), rng.normal(size=(T, dm)), rng.normal(size=(dm, dv)),
            rng.normal(size=(dv, dm)), rng.normal(size=(T, dm)))


def test_memplus_backward_matches_autograd(orc):
    """dy, dx, dW1, dW2 equal torch autograd (fp64) of <dout, (y ⊙ silu(x W1)) W2>;
    x, W1 and W2 travel as bf16 (exact decoding)."""
    y, x, W1, W2, dout = _memplus_inputs(21)
    xb, W1b, W2b = (torch.from_numpy(a).to(torch.bfloat16) for a in (x, W1, W2))
    r = orc.memplus_backward(y, xb, W1b, W2b, dout)
    yt = torch.tensor(y, requires_grad=True)
    xt, W1t, W2t = (a.double().requires_grad_(True) for a in (xb, W1b, W2b))
    out = (yt * torch.nn.functional.silu(xt @ W1t)) @ W2t
    (out * torch.from_numpy(dout)).sum().backward()
    for key, t in (("dy", yt), ("dx", xt), ("dW1", W1t), ("dW2", W2t)):
        np.testing.assert_allclose(r[key], t.grad.numpy(), rtol=1e-12, atol=1e-12, err_msg=key)


def test_memplus_backward_finite_differences(orc):
    """Central differences of <dout, memplus(y, x, W1, W2)> (the oracle's own
    forward, pinned above) on every entry of small inputs."""
    y, x, W1, W2, dout = _memplus_inputs(22, T=3, dm=4, dv=3)
    r = orc.memplus_backward(y, x, W1, W2, dout)
    h = 1e-6

    def f(y_, x_, W1_, W2_):
        return float(np.sum(orc.memplus(y_, x_, W1_, W2_) * dout))

    args = [y, x, W1, W2]
    for pos, key in ((0, "dy"), (1, "dx"), (2, "dW1"), (3, "dW2")):
        num = np.empty_like(args[pos])
        for i in np.ndindex(args[pos].shape):
            up = [a.copy() for a in args]
            dn = [a.copy() for a in args]
            up[pos][i] += h
            dn[pos][i] -= h
            num[i] = (f(*up) - f(*dn)) / (2 * h)
        np.testing.assert_allclose(r[key], num, rtol=1e-6, atol=1e-7, err_msg=key)


def test_memplus_backward_zero_gate(orc):
    """W1 = 0: a = 0, silu(0) = 0, silu'(0) = 1/2, so dy = 0, dW2 = 0 and
    da = (dout W2^T) ⊙ y / 2 (dW1 = x^T da, dx = da W1^T = 0)."""
    y, x, _, W2, dout = _memplus_inputs(23)
    W1 = np.zeros((x.shape[1], y.shape[1]))
    r = orc.memplus_backward(y, x, W1, W2, dout)
    assert np.all(r["dy"] == 0.0) and np.all(r["dW2"] == 0.0) and np.all(r["dx"] == 0.0)
    da = (dout @ W2.T) * y * 0.5
    np.testing.assert_allclose(r["dW1"], x.T @ da, rtol=1e-13, atol=1e-14)


def test_qproj_and_backward(orc):
    """q = x Wq is numpy's matmul; its backward equals autograd (bf16 inputs)."""
    rng = np.random.default_rng(24)
    x, Wq, dq = rng.normal(size=(5, 6)), rng.normal(size=(6, 8)), rng.normal(size=(5, 8))
    xb, Wqb = torch.from_numpy(x).to(torch.bfloat16), torch.from_numpy(Wq).to(torch.bfloat16)
    q = orc.qproj(xb, Wqb)
    np.testing.assert_allclose(q, xb.double().numpy() @ Wqb.double().numpy(), rtol=1e-13)
    xt, Wt = xb.double().requires_grad_(True), Wqb.double().requires_grad_(True)
    ((xt @ Wt) * torch.from_numpy(dq)).sum().backward()
    r = orc.qproj_backward(xb, Wqb, dq)
    np.testing.assert_allclose(r["dWq"], Wt.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["dx"], xt.grad.numpy(), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# sparse optimiser step on the touched rows
# --------------------------------------------------------------------------

def test_sparse_sgd_equals_dense_sgd_with_zero_rows(orc):
    """Sparse SGD equals torch's dense SGD step whose gradient is zero on the
    untouched rows."""
    rng = np.random.default_rng(31)
    table, rows = rng.normal(size=(20, 6)), np.array([3, 7, 11, 19])
    grads = rng.normal(size=(4, 6))
    p = torch.tensor(table, requires_grad=True)
    dense = np.zeros_like(table)
    dense[rows] = grads
    p.grad = torch.from_numpy(dense)
    torch.optim.SGD([p], lr=0.05).step()
    np.testing.assert_allclose(orc.sparse_sgd(table, rows, grads, 0.05), p.detach().numpy(),
                               rtol=0, atol=1e-15)


def test_sparse_adam_equals_torch_sparse_adam(orc):
    """Three steps of the touched-rows Adam equal torch.optim.SparseAdam fed
    the same sparse gradients (different rows each step).  torch applies eps
    after folding the bias corrections into the step size (eps scaled by
    sqrt(1 - beta2^t) relative to the oracle's m_hat / (sqrt(v_hat) + eps));
    a negligible eps makes the two forms coincide."""
    rng = np.random.default_rng(32)
    table = rng.normal(size=(16, 5))
    p = torch.nn.Parameter(torch.tensor(table))
    opt = torch.optim.SparseAdam([p], lr=0.01, betas=(0.9, 0.99), eps=1e-30)
    t, m, v = table, np.zeros_like(table), np.zeros_like(table)
    for step, rows in enumerate(([1, 4, 9], [4, 5], [0, 9, 15]), start=1):
        rows = np.array(rows)
        grads = rng.normal(size=(len(rows), 5))
        with torch.sparse.check_sparse_tensor_invariants():
            p.grad = torch.sparse_coo_tensor(torch.from_numpy(rows)[None],
                                             torch.from_numpy(grads), (16, 5))
        opt.step()
        t, m, v = orc.sparse_adam(t, m, v, rows, grads, 0.01, 0.9, 0.99, 1e-30, step)
        np.testing.assert_allclose(t, p.detach().numpy(), rtol=1e-12, atol=1e-14)
    untouched = np.setdiff1d(np.arange(16), [0, 1, 4, 5, 9, 15])
    np.testing.assert_array_equal(t[untouched], table[untouched])


def test_sparse_adam_first_step_closed_form(orc):
    """Step 1 from zero moments: m_hat = g and v_hat = g^2, so the update is
    lr * g / (|g| + eps) on the touched rows."""
    rng = np.random.default_rng(33)
    table, rows = rng.normal(size=(10, 4)), np.array([2, 6])
    g = rng.normal(size=(2, 4))
    t, m, v = orc.sparse_adam(table, np.zeros_like(table), np.zeros_like(table), rows, g,
                              0.1, 0.9, 0.999, 0.5, 1)
    ref = table.copy()
    ref[rows] -= 0.1 * g / (np.abs(g) + 0.5)
    np.testing.assert_allclose(t, ref, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# Engram ("Conditional Memory via Scalable Lookup" review): hashed n-gram
# rows and the context gate.  The page names independent hash functions per
# order and head but not the functions, so the hash is pinned by what the
# page does fix: each head reads its own table, a row depends on its n-gram
# window alone, equal n-grams give equal rows, and the heads are independent.
# --------------------------------------------------------------------------

_ORDERS, _K = [2, 3], 2
_SEEDS = [0x1234, 0xBEEF, 0x51ED, 0xC0DE]
_M = [1009, 1013, 997, 1019]


def test_engram_rows_stay_in_their_heads_table(orc):
    tok = np.random.default_rng(40).integers(0, 50000, (3, 200))
    rows = orc.engram_rows(tok, _ORDERS, _K, _SEEDS, _M)
    off = np.concatenate([[0], np.cumsum(_M)[:-1]])
    assert rows.shape == (600, 4)
    assert np.all(rows >= off) and np.all(rows < off + np.array(_M))


def test_engram_row_depends_only_on_its_window(orc):
    """Changing a token outside positions p-n+1..p leaves the order-n rows
    at p alone; changing one inside moves them (up to a 1/M collision)."""
    rng = np.random.default_rng(41)
    tok = rng.integers(0, 50000, (1, 64))
    base = orc.engram_rows(tok, _ORDERS, _K, _SEEDS, _M)
    p = 40
    moved = 0
    for o, n in enumerate(_ORDERS):
        cols = slice(o * _K, (o + 1) * _K)
        for q in (p - n, p + 1):  # just outside the window
            t2 = tok.copy()
            t2[0, q] += 1
            np.testing.assert_array_equal(orc.engram_rows(t2, _ORDERS, _K, _SEEDS, _M)[p, cols],
                                          base[p, cols])
        for q in range(p - n + 1, p + 1):  # inside it
            t2 = tok.copy()
            t2[0, q] += 1
            moved += int(np.any(orc.engram_rows(t2, _ORDERS, _K, _SEEDS, _M)[p, cols]
                                != base[p, cols]))
    assert moved == sum(_ORDERS)


def test_engram_equal_ngrams_equal_rows(orc):
    """The same n-gram planted at other positions and in another sequence
    reads the same rows; a bigram that agrees only in its last token does
    not."""
    rng = np.random.default_rng(42)
    tok = rng.integers(0, 50000, (2, 50))
    tok[0, 10:13] = tok[1, 30:33] = [7, 8, 9]
    rows = orc.engram_rows(tok, _ORDERS, _K, _SEEDS, _M).reshape(2, 50, -1)
    np.testing.assert_array_equal(rows[0, 12], rows[1, 32])      # 2- and 3-gram (7,8,9)
    np.testing.assert_array_equal(rows[0, 11, :_K], rows[1, 31, :_K])  # bigram (7,8)
    tok[1, 31] = 6                                                # (6,9) vs (8,9)
    rows2 = orc.engram_rows(tok, _ORDERS, _K, _SEEDS, _M).reshape(2, 50, -1)
    assert np.any(rows2[1, 32, :_K] != rows[0, 12, :_K])


def test_engram_sequence_start_reads_the_pad_id(orc):
    """Before a sequence's first token the n-gram reads the pad id: position
    0 of a sequence equals position 1 of the same sequence with the pad id
    (-1 as a 32-bit token) put in front, for every order whose window ends
    there -- and sequences do not leak into each other."""
    rng = np.random.default_rng(43)
    s = rng.integers(0, 50000, 30)
    a = orc.engram_rows(s[None], _ORDERS, _K, _SEEDS, _M)
    padded = np.concatenate([[-1, -1], s])[None]
    b = orc.engram_rows(padded, _ORDERS, _K, _SEEDS, _M)
    np.testing.assert_array_equal(a, b[2:])
    two = orc.engram_rows(np.stack([s, s]), _ORDERS, _K, _SEEDS, _M)
    np.testing.assert_array_equal(two[:30], two[30:])


def test_engram_rows_fill_the_table_evenly(orc):
    """Distinct bigrams spread over a head's M rows like uniform draws
    (chi-square statistic within 6 standard deviations of its mean)."""
    M = 1009
    tok = np.random.default_rng(44).integers(0, 2 ** 31 - 1, (1, 200000))
    rows = orc.engram_rows(tok, [2], 1, [99], [M])[1:, 0]
    cnt = np.bincount(rows, minlength=M)
    exp = len(rows) / M
    chi2 = float(((cnt - exp) ** 2 / exp).sum())
    assert abs(chi2 - (M - 1)) < 6 * math.sqrt(2 * (M - 1))


def test_engram_heads_hash_independently(orc):
    """Two heads with the same table size: the same bigrams land in the same
    row of both about 1/M of the time, as independent hashes would."""
    M = 1009
    tok = np.random.default_rng(45).integers(0, 50000, (1, 100000))
    rows = orc.engram_rows(tok, [2], 2, [5, 6], [M, M])
    same = np.mean(rows[:, 0] == rows[:, 1] - M)
    assert abs(same - 1 / M) < 6 * math.sqrt(1 / M / len(rows))


def test_engram_gate_closed_forms(orc):
    """h along e: <RMSNorm(h), RMSNorm(e)> = d, so alpha = sigmoid(sqrt(d));
    h against e: sigmoid(-sqrt(d)); h orthogonal to e: 1/2.  Large values
    make the eps of the norm negligible."""
    d = 64
    E = np.zeros((3, d))
    E[0, :] = 300.0
    E[1, : d // 2] = 500.0
    E[2, d // 2:] = 500.0
    rows = np.array([[0], [0], [1]])
    h = np.stack([np.full(d, 100.0), np.full(d, -100.0), np.r_[np.zeros(d // 2),
                                                              np.full(d // 2, 100.0)]])
    r = orc.engram_gate(rows, E, h)
    sig = lambda z: 1 / (1 + math.exp(-z))
    np.testing.assert_allclose(r["alpha"], [sig(math.sqrt(d)), sig(-math.sqrt(d)), 0.5],
                               rtol=1e-9)
    np.testing.assert_allclose(r["v"], r["alpha"][:, None] * r["e"], rtol=1e-15)


def test_engram_gate_matches_library(orc):
    """torch's embedding_bag (sum) and rms_norm in fp64 on random rows."""
    rng = np.random.default_rng(46)
    T, HK, d, n_rows = 20, 6, 48, 300
    E = rng.normal(size=(n_rows, d))
    rows = rng.integers(0, n_rows, (T, HK))
    h = rng.normal(size=(T, d))
    r = orc.engram_gate(rows, E, h)
    Et = torch.tensor(E)
    e = torch.nn.functional.embedding_bag(torch.tensor(rows), Et, mode="sum")
    ht = torch.tensor(h)
    nh = torch.nn.functional.rms_norm(ht, (d,), eps=orc.ENGRAM_EPS)
    ne = torch.nn.functional.rms_norm(e, (d,), eps=orc.ENGRAM_EPS)
    alpha = torch.sigmoid((nh * ne).sum(-1) / math.sqrt(d))
    np.testing.assert_allclose(r["e"], e.numpy(), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(r["alpha"], alpha.numpy(), rtol=1e-12)
    np.testing.assert_allclose(r["v"], (alpha[:, None] * e).numpy(), rtol=1e-12, atol=1e-13)


def test_engram_rows_golden(orc):
    """tests/golden/engram_rows.json (written by make_engram_rows.py from the
    oracle) freezes the hash definition; the stored rows are also re-derived
    here from the definition in include/pkm.h with Python integers (64-bit
    wrap-around written out), which checks the C oracle's unsigned
    arithmetic, seeds at both ends of the 64-bit range and a one-row head."""
    g = json.load(open(os.path.join(GOLDEN, "engram_rows.json")))
    seeds = [int(s) for s in g["seeds"]]
    rows = orc.engram_rows(g["tokens"], g["orders"], g["K"], seeds, g["M"])
    np.testing.assert_array_equal(rows, np.array(g["rows"]))
    mask = (1 << 64) - 1
    off = np.concatenate([[0], np.cumsum(g["M"])[:-1]])
    L = len(g["tokens"][0])
    for s, seq in enumerate(g["tokens"]):
        for p in range(L):
            for o, n in enumerate(g["orders"]):
                for k in range(g["K"]):
                    j = o * g["K"] + k
                    h = seeds[j]
                    for q in range(p - n + 1, p + 1):
                        x = seq[q] & 0xFFFFFFFF if q >= 0 else 0xFFFFFFFF
                        h = ((h ^ x) * 0x9E3779B97F4A7C15) & mask
                        h ^= h >> 32
                    assert rows[s * L + p, j] == off[j] + h % g["M"][j]
