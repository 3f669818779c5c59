"""GPU parity of the forward path against the CPU oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

from parity import RTOL, W_RTOL, close, forward_reference, weights_close

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


def run_forward(w, inp=None, sample=None, max_exempt=0.01):
    """Run the GPU forward of workload ``w`` and check it against the oracle
    on the tokens ``sample`` (all tokens by default).  At most a fraction
    ``max_exempt`` of the (token, head) selections may differ from the
    oracle's, each within the tie rule."""
    import oracle

    if inp is None:
        inp = make_inputs(w, "cuda")
    mp = w.memplus
    out, idx, wts = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k,
                                    x=inp.get("x") if mp else None,
                                    W1=inp.get("W1") if mp else None,
                                    W2=inp.get("W2") if mp else None)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    if sample is None:
        sample = torch.arange(w.T)
    sample = torch.as_tensor(sample, dtype=torch.long)
    sd = sample.to("cuda")
    idx_g = idx[sd].cpu().numpy().astype(np.int64)
    rows = np.unique(idx_g)
    table_rows = inp["values"][torch.from_numpy(rows).to("cuda")].cpu()
    ref = forward_reference(inp["query"][sd].cpu(), inp["subkeys"].cpu(), w.k, idx_g,
                            table_rows, rows, w.n_sub,
                            x=inp["x"][sd].cpu() if mp else None,
                            W1=inp["W1"].cpu() if mp else None,
                            W2=inp["W2"].cpu() if mp else None)
    weights_close(wts[sd].cpu().numpy(), ref["w_ref"], W_RTOL[w.dtype])
    err = close(out[sd].float().cpu().numpy(), ref["out_ref"], RTOL[w.dtype], "out")
    n_th = len(sample) * w.H
    assert ref["exempt"] <= max(1, max_exempt * n_th), f"{ref['exempt']} tie exemptions of {n_th}"
    return dict(ref=ref, idx=idx_g, err=err, inp=inp)


SMALL = [
    # name, T, H, d_half, n_sub, k, d_v, dtype
    ("bf16-ragged", 300, 2, 64, 64, 16, 128, "bf16"),
    ("bf16-k32-odd-n", 129, 3, 128, 100, 32, 64, "bf16"),
    ("bf16-minimal", 1, 1, 8, 3, 1, 8, "bf16"),
    ("bf16-wide", 37, 4, 512, 300, 32, 2048, "bf16"),
    ("tc-two-chunks", 300, 2, 128, 512, 16, 64, "bf16"),
    ("tc-k32-many-tiles", 1000, 1, 64, 1024, 32, 128, "bf16"),
    ("tc-k1", 130, 2, 64, 256, 1, 16, "bf16"),
    # five chunks, the last one ragged: prefix pass over four, main pass over five
    ("tc-prefix-ragged", 200, 2, 64, 1100, 32, 32, "bf16"),
    # n % 4 != 0 takes the SIMT scoring path even with n >= 256
    ("bf16-n-mod4", 90, 2, 64, 258, 8, 16, "bf16"),
    ("f32-k64", 70, 2, 32, 64, 64, 40, "f32"),
    ("f32-k-equals-n", 33, 1, 16, 5, 5, 24, "f32"),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_forward_small(case):
    name, T, H, dh, n, k, dv, dt = case
    w = WORKLOADS["pkm"].scaled(name=name, T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv, dtype=dt,
                                seed=sum(map(ord, name)))
    run_forward(w)



# Batches of more than 64 tokens with bf16, d_half % 64 == 0, n >= 256,
# n % 4 == 0 and k <= 32 run the one-kernel selection (query norms, scores,
# per-half top-k, k x k combine and softmax in one launch; one CTA per (token
# tile, head, half), the second CTA of a (tile, head) to finish combines; k = 32
# skips sorting the combine's first group, the grid's already ordered first row).
FUSED = [
    # name, T, H, d_half, n_sub, k, d_v
    ("fused-k32-ragged-tile", 333, 2, 64, 512, 32, 64),
    ("fused-k7-three-heads", 200, 3, 128, 768, 7, 32),
    ("fused-ragged-chunk", 129, 1, 192, 1100, 32, 16),
    ("fused-k1", 65, 2, 64, 256, 1, 16),
    ("fused-wide-query", 160, 2, 512, 2048, 32, 32),
    ("fused-many-chunks", 130, 1, 64, 4096, 32, 16),
    ("fused-k31", 300, 1, 256, 300, 31, 24),
]


@pytest.mark.parametrize("case", FUSED, ids=[c[0] for c in FUSED])
def test_forward_fused_selection(case):
    name, T, H, dh, n, k, dv = case
    w = WORKLOADS["pkm"].scaled(name=name, T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv,
                                dtype="bf16", seed=sum(map(ord, name)))
    run_forward(w)


# Batches of at most 32 tokens (decode steps) run the one-kernel small-batch
# selection: each 256-column chunk of a (head, half) in its own CTA (sub-key
# and query norms from the staged tiles, the chunk's scores sorted per token
# across a warp), the last CTA of a half merging the chunks' lists and the
# last half of a head combining; 33..64 tokens keep the column-split kernel
# with per-thread top-k.
SMALL_T = [
    # name, T, H, d_half, n_sub, k, d_v
    ("small-t8", 8, 4, 64, 1024, 32, 64),
    ("small-t32-ragged-chunk", 32, 2, 128, 300, 16, 32),
    ("small-t1-k1", 1, 1, 64, 256, 1, 16),
    ("small-t5-k7", 5, 3, 192, 700, 7, 24),
    ("small-t3-32-chunks", 3, 2, 64, 8192, 32, 8),
    ("small-t8-wide", 8, 2, 512, 4096, 32, 32),
    ("small-t17-k31-ragged", 17, 1, 256, 1100, 31, 16),
    ("split-t40", 40, 2, 64, 512, 32, 32),
    # the first and last batch sizes of the column-split path
    ("split-t33", 33, 2, 64, 512, 32, 32),
    ("split-t64-ragged", 64, 1, 128, 300, 16, 48),
]


@pytest.mark.parametrize("case", SMALL_T, ids=[c[0] for c in SMALL_T])
def test_forward_small_batches(case):
    name, T, H, dh, n, k, dv = case
    w = WORKLOADS["pkm"].scaled(name=name, T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv,
                                dtype="bf16", seed=sum(map(ord, name)))
    run_forward(w)


def test_forward_fused_launches():
    """A batch on the one-kernel selection launches three kernels in all:
    the sub-key norms, the selection and the bag gather."""
    w = WORKLOADS["pkm"].scaled(T=300, H=2, d_half=64, n_sub=512, k=32, d_v=64)
    inp = make_inputs(w, "cuda")
    lib = skv.load()
    skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    torch.cuda.synchronize()
    c0 = lib.pkm_launch_count()
    skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    torch.cuda.synchronize()
    assert lib.pkm_launch_count() - c0 == 3
    assert skv.device_error() == 0

def test_forward_small_launches():
    """A decode-sized batch launches three kernels in all: the one-kernel
    selection and the two steps of the row-group gather."""
    w = WORKLOADS["pkm"].scaled(T=8, H=2, d_half=64, n_sub=512, k=32, d_v=64)
    inp = make_inputs(w, "cuda")
    lib = skv.load()
    skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    torch.cuda.synchronize()
    c0 = lib.pkm_launch_count()
    skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    torch.cuda.synchronize()
    assert lib.pkm_launch_count() - c0 == 3
    assert skv.device_error() == 0


@pytest.mark.parametrize("sign", [1.0, -1.0], ids=["aligned", "anti-aligned"])
def test_forward_extreme_scores(sign):
    """Queries (anti-)aligned with every sub-key of their (head, half): the
    scores sit around +/-6.5, so the group maxima fall outside the histogram
    range of the prefix pass (its bound saturates at the top bin, or is empty
    at the bottom); the selection must still be exact.  A shared direction
    also crowds the scores, so near-ties (each still within the tie rule)
    are more frequent than on isotropic inputs: up to 3% are allowed."""
    w = WORKLOADS["pkm"].scaled(name="extreme", T=260, H=2, d_half=512, n_sub=512, k=32, d_v=32,
                                seed=77)
    inp = make_inputs(w, "cuda")
    g = torch.Generator().manual_seed(78)
    e = torch.randn(w.H, 2, w.d_half, generator=g)
    e = e / e.norm(dim=-1, keepdim=True)
    q = inp["query"].float().cpu() + sign * 10.0 * e.unsqueeze(0)
    K = inp["subkeys"].float().cpu() + 1.0 * e.unsqueeze(2)
    inp["query"] = q.to(torch.bfloat16).cuda()
    inp["subkeys"] = K.to(torch.bfloat16).cuda()
    run_forward(w, inp=inp, max_exempt=0.03)


def test_forward_zipf_scores():
    """Sub-keys biased towards a shared direction (the training workload's
    Zipf popularity) at a small size: a heavy upper tail of scores."""
    w = WORKLOADS["train"].scaled(name="zipf-small", T=400, H=2, d_half=128, n_sub=1024, k=32,
                                  d_v=32, train=False)
    run_forward(w)


def test_forward_tiny_workload_and_bruteforce():
    """The tiny fp32 workload end to end; the selection also equals the
    brute-force top-k over all 1024 full keys."""
    import oracle

    w = WORKLOADS["tiny"]
    r = run_forward(w)
    bidx, _ = oracle.bruteforce_select(r["inp"]["query"].cpu(), r["inp"]["subkeys"].cpu(), w.k)
    assert r["ref"]["exempt"] == 0
    np.testing.assert_array_equal(r["idx"], bidx)


MEMPLUS = [
    # T, H, d_half, n_sub, k, d_v, d_model
    (200, 2, 64, 64, 8, 256, 128),     # output projection N < tile
    (300, 1, 128, 256, 16, 512, 320),  # ragged N, tensor-core scoring
    (50, 2, 64, 16, 4, 80, 40),        # K below one k-block: SIMT GEMM
    (8, 4, 128, 256, 32, 1024, 1024),  # decode-sized: the few-row GEMM
    (64, 1, 64, 256, 8, 264, 136),     # few-row GEMM, ragged column strips
    (65, 1, 64, 256, 8, 264, 136),     # just past the few-row GEMM: tensor cores
]


@pytest.mark.parametrize("shape", MEMPLUS)
def test_forward_memplus_small(shape):
    T, H, dh, n, k, dv, dm = shape
    w = WORKLOADS["memplus"].scaled(T=T, H=H, d_half=dh, n_sub=n, k=k, d_v=dv, d_model=dm,
                                    seed=T + dv)
    run_forward(w)


def test_forward_empty_batch():
    w = WORKLOADS["pkm"].scaled(T=0, H=2, d_half=64, n_sub=16, k=4, d_v=64)
    inp = make_inputs(w, "cuda")
    out, idx, wts = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    assert out.shape == (0, 64)


def test_forward_deterministic():
    w = WORKLOADS["pkm"].scaled(T=257, H=2, d_half=64, n_sub=128, k=32, d_v=256)
    inp = make_inputs(w, "cuda")
    a = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    b = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ------------------------------------------------------------ bag gather --

BAGS = [(1, 1, 8, "bf16"), (513, 128, 2048, "bf16"), (77, 33, 1024, "bf16"),
        (50, 7, 24, "f32"), (31, 128, 4096, "bf16"), (200, 5, 8, "f32"),
        (301, 16, 512, "bf16"), (64, 9, 256, "f32"), (40, 3, 1024, "f32"),
        (5, 2, 8192, "bf16"), (1, 130, 512, "bf16")]


@pytest.mark.parametrize("n_bags,B,d,dt", BAGS)
@pytest.mark.parametrize("gate", [False, True])
def test_embbag_forward(n_bags, B, d, dt, gate):
    import oracle

    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    n_rows = 1000
    g = torch.Generator().manual_seed(n_bags * 7 + B)
    table = (torch.randn(n_rows, d, generator=g) * 0.02).to(tdt).cuda()
    idx, w = random_bags(n_bags, B, n_rows, seed=B + d)
    gt = torch.randn(n_bags, d, generator=g).to(tdt).cuda() if gate else None
    out = skv.embbag_forward(table, idx.cuda(), w.cuda(), gate=gt)
    ref = oracle.bag(idx.numpy(), w.double().numpy(), table.cpu())
    if gate:
        ref = ref * gt.double().cpu().numpy()
    close(out.double().cpu().numpy(), ref, RTOL[dt], "embbag")


def test_embbag_bad_index_sets_status():
    table = torch.randn(10, 16, dtype=torch.bfloat16, device="cuda")
    idx = torch.tensor([[0, 1, 10], [2, -1, 3]], dtype=torch.int32, device="cuda")
    w = torch.full((2, 3), 0.5, device="cuda")
    out = skv.embbag_forward(table, idx, w)
    assert skv.device_error() == 4  # PKM_ERR_DEVICE
    assert skv.device_error() == 0  # cleared on read
    ref = 0.5 * (table[0].float() + table[1].float())
    torch.testing.assert_close(out[0].float(), ref, rtol=2e-2, atol=1e-2)


def test_embbag_bad_index_wide_rows():
    """Bad row ids among many good ones in rows of 1 KiB: each bad id is
    skipped and reported; the other rows of its bag still sum."""
    g = torch.Generator().manual_seed(5)
    table = torch.randn(50, 512, generator=g).to(torch.bfloat16).cuda()
    idx = torch.tensor([[0, 1, 50], [2, -7, 3], [4, 5, 6]], dtype=torch.int32, device="cuda")
    w = torch.full((3, 3), 0.5, device="cuda")
    out = skv.embbag_forward(table, idx, w)
    assert skv.device_error() == 4  # PKM_ERR_DEVICE
    ref = 0.5 * torch.stack([table[0].float() + table[1].float(),
                             table[2].float() + table[3].float(),
                             table[4].float() + table[5].float() + table[6].float()])
    torch.testing.assert_close(out.float(), ref, rtol=2e-2, atol=1e-2)


def test_embbag_row_order_sum():
    """The gather sums each bag's rows in order j = 0 .. B-1 in fp32 and
    rounds once: against a sequential fp32 sum done here (fused and separate
    multiply-adds differ by at most one rounding per row)."""
    g = torch.Generator().manual_seed(6)
    n_bags, B, d = 9, 40, 1024
    table = torch.randn(300, d, generator=g).to(torch.bfloat16)
    idx, w = random_bags(n_bags, B, 300, seed=7)
    out = skv.embbag_forward(table.cuda(), idx.cuda(), w.cuda())
    ref = torch.zeros(n_bags, d)
    tf = table.float()
    for j in range(B):
        ref = ref + w[:, j:j + 1] * tf[idx[:, j].long()]
    torch.testing.assert_close(out.float().cpu(), ref.to(torch.bfloat16).float(), rtol=1e-2,
                               atol=1e-3)


# ------------------------------------------------- full-size workloads --

def _sample(T, m, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.randperm(T, generator=g)[: m - 2]
    return torch.cat([torch.tensor([0, T - 1]), s]).sort().values


def test_forward_pkm_full_size_sampled():
    w = WORKLOADS["pkm"]
    run_forward(w, sample=_sample(w.T, 64, 1))


def test_forward_memplus_full_size_sampled():
    w = WORKLOADS["memplus"]
    r = run_forward(w, sample=_sample(w.T, 32, 2))
    del r
    torch.cuda.empty_cache()


def test_decode_steps():
    """Decode-shaped lookups (8 tokens per step) against the 16.8M-key tables."""
    from sparse_key_value_b200.inputs import decode_step_inputs

    w = WORKLOADS["decode"]
    base = make_inputs(w.scaled(T=8), "cuda")
    for step in (0, 1, 255):
        inp = dict(base)
        inp.update(decode_step_inputs(w, step, "cuda"))
        run_forward(w, inp=inp)
    del base
    torch.cuda.empty_cache()


# The selection at the largest supported sizes: n_sub^2 < 2^31 allows n_sub =
# 46340 (a multiple of 4, so the tensor-core selection takes it: 363 chunks,
# the last one ragged), and d_half = 2048 is the widest query half (32
# k-blocks per chunk); two token tiles, the second ragged
@pytest.mark.parametrize("n,dh", [(46340, 64), (1024, 2048)], ids=["n-46340", "dh-2048"])
def test_select_maximum_sizes(n, dh):
    import oracle
    from parity import check_selection, weights_close, W_RTOL

    w = WORKLOADS["pkm"].scaled(name=f"max-{n}-{dh}", T=130, H=1, d_half=dh, n_sub=n, k=32,
                                d_v=8, seed=n + dh)
    inp = make_inputs(w, "cuda", with_values=False)
    idx, wts = skv.pkm_select(inp["query"], inp["subkeys"], w.k, d_v=w.d_v)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    q, K = inp["query"].cpu(), inp["subkeys"].cpu()
    idx_o, S_o, w_o, _ = oracle.pkm_select(q, K, w.k)
    s_half = oracle.half_scores(q, K)
    G = idx.cpu().numpy().astype(np.int64)
    exempt = check_selection(G, idx_o, s_half, n)
    assert exempt <= 1, f"{exempt} tie exemptions"
    weights_close(wts.cpu().numpy(), oracle.softmax(oracle.full_scores(s_half, G, n)),
                  W_RTOL["bf16"])
