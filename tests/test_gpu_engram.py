"""GPU parity of the Engram lookup ("Conditional Memory via Scalable Lookup"
review, "희소 검색" and "핵심 수식" 1-2) against the CPU oracle, through the C
ABI: hashed n-gram rows bit-exact; the gate alpha within 1e-4 absolute (fp32
sums over d of products of bf16 h and the fp32 row sum: the logit
sqrt(d) * cos carries an error of about sqrt(d) * 2e-6, and sigmoid' <= 1/4);
the summed rows e and v = alpha * e under the bf16/fp32 output rule."""

import numpy as np
import pytest
import torch

from parity import RTOL, close

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import ENGRAM, make_engram_inputs  # noqa: E402

ALPHA_ATOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    yield
    assert skv.device_error() == 0


def _check(w, inp, sample=None):
    import oracle

    r = skv.engram_forward(inp["tokens"], inp["table"], inp["h"], w.orders, w.K, w.seeds,
                           w.rows_per_head, rows=True, e=True)
    torch.cuda.synchronize()
    ref_rows = oracle.engram_rows(inp["tokens"].cpu().numpy(), w.orders, w.K, w.seeds,
                                  w.rows_per_head)
    np.testing.assert_array_equal(r["rows"].cpu().numpy().astype(np.int64), ref_rows)
    if sample is None:
        sample = np.arange(w.T)
    rows = ref_rows[sample]
    uniq, inv = np.unique(rows, return_inverse=True)
    E = inp["table"][torch.from_numpy(uniq).cuda()].cpu()
    ref = oracle.engram_gate(inv.reshape(rows.shape), E, inp["h"][torch.from_numpy(sample).cuda()]
                             .cpu())
    sd = torch.from_numpy(sample).cuda()
    np.testing.assert_allclose(r["alpha"][sd].cpu().numpy(), ref["alpha"], rtol=0,
                               atol=ALPHA_ATOL)
    close(r["e"][sd].double().cpu().numpy(), ref["e"], RTOL[w.dtype], "e")
    close(r["v"][sd].double().cpu().numpy(), ref["v"], RTOL[w.dtype], "v")
    return r


PRIMES = (5003, 5009, 5011, 5021, 5023, 5039, 5051, 5059)
CASES = [
    # name, n_seq, L, orders, K, d, dtype
    ("bf16-d256", 3, 100, (2, 3), 2, 256, "bf16"),
    ("bf16-d1024", 2, 300, (2, 3), 4, 1024, "bf16"),
    ("bf16-d2048", 2, 50, (2, 3), 4, 2048, "bf16"),
    ("bf16-d8192", 1, 20, (2,), 1, 8192, "bf16"),
    ("bf16-d136-ragged-columns", 2, 40, (1, 2, 3), 2, 136, "bf16"),
    ("f32-d512", 2, 64, (1, 2, 3), 3, 512, "f32"),
    ("f32-d4096", 1, 10, (4,), 2, 4096, "f32"),
    ("single-token-sequences", 5, 1, (1, 2, 8), 1, 64, "bf16"),
    ("64-heads", 1, 40, (1, 2, 3, 4, 5, 6, 7, 8), 8, 64, "bf16"),
    ("d8-one-column", 3, 17, (2, 3), 1, 8, "bf16"),
    ("unigram-only-f32", 4, 33, (1,), 5, 40, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_engram_matches_oracle(case):
    name, n_seq, L, orders, K, d, dt = case
    heads = len(orders) * K
    M = tuple(PRIMES[j % len(PRIMES)] + 2 * (j // len(PRIMES)) for j in range(heads))
    if name == "d8-one-column":
        M = (1,) + M[1:]  # a one-row head table: every n-gram reads its only row
    w = ENGRAM.scaled(name=name, n_seq=n_seq, L=L, orders=orders, K=K, rows_per_head=M, d=d,
                      dtype=dt, seed=sum(map(ord, name)))
    inp = make_engram_inputs(w, "cuda")
    _check(w, inp)


def test_engram_extreme_token_ids_and_repeats():
    """Ids up to 2^31-1 (all 32 bits hashed), repeated n-grams across
    sequences and positions (equal rows on both sides)."""
    w = ENGRAM.scaled(n_seq=2, L=64, rows_per_head=PRIMES, d=128, seed=7)
    inp = make_engram_inputs(w, "cuda")
    tok = inp["tokens"].cpu()
    tok[0, :8] = torch.tensor([2 ** 31 - 1, 0, 1, 2 ** 31 - 2, 5, 5, 5, 5], dtype=torch.int32)
    tok[1, 20:28] = tok[0, :8]
    inp["tokens"] = tok.cuda()
    r = _check(w, inp)
    rows = r["rows"].cpu().view(2, 64, -1)
    assert torch.equal(rows[0, 7], rows[1, 27])


def test_engram_alpha_closed_forms():
    """h along e gives sigmoid(sqrt(d)), h against e sigmoid(-sqrt(d))."""
    import math

    w = ENGRAM.scaled(n_seq=1, L=4, orders=(1,), K=1, rows_per_head=(7,), d=256, seed=8)
    inp = make_engram_inputs(w, "cuda")
    r0 = skv.engram_forward(inp["tokens"], inp["table"], inp["h"], w.orders, w.K, w.seeds,
                            w.rows_per_head, e=True)
    e = r0["e"].float()
    h = torch.cat([e[:2] * 50.0, -e[2:] * 50.0]).to(torch.bfloat16)
    r = skv.engram_forward(inp["tokens"], inp["table"], h, w.orders, w.K, w.seeds,
                           w.rows_per_head)
    torch.cuda.synchronize()
    s = 1 / (1 + math.exp(-math.sqrt(w.d)))
    np.testing.assert_allclose(r["alpha"].cpu().numpy(), [s, s, 1 - s, 1 - s], atol=1e-3)


def test_engram_empty_batch():
    w = ENGRAM.scaled(n_seq=0, L=16, rows_per_head=PRIMES, d=64)
    inp = make_engram_inputs(w, "cuda")
    r = skv.engram_forward(inp["tokens"], inp["table"], inp["h"], w.orders, w.K, w.seeds,
                           w.rows_per_head)
    assert r["v"].shape == (0, 64)


def test_engram_deterministic():
    w = ENGRAM.scaled(n_seq=2, L=128, rows_per_head=PRIMES, d=512, seed=9)
    inp = make_engram_inputs(w, "cuda")
    a = skv.engram_forward(inp["tokens"], inp["table"], inp["h"], w.orders, w.K, w.seeds,
                           w.rows_per_head)
    b = skv.engram_forward(inp["tokens"], inp["table"], inp["h"], w.orders, w.K, w.seeds,
                           w.rows_per_head)
    assert torch.equal(a["v"], b["v"]) and torch.equal(a["alpha"], b["alpha"])


def test_engram_full_size_sampled():
    """The benchmarked configuration (16,384 tokens, 8 heads, 17 GB of
    tables): every row id exact, the gate and outputs on sampled tokens."""
    w = ENGRAM
    inp = make_engram_inputs(w, "cuda")
    g = torch.Generator().manual_seed(3)
    sample = np.sort(np.concatenate([[0, w.L - 1, w.T - 1],
                                     torch.randperm(w.T, generator=g)[:61].numpy()]))
    _check(w, inp, sample=sample)
    del inp
    torch.cuda.empty_cache()
