"""Properties of the synthetic workloads (CPU, no GPU needed)."""

import math

import pytest
import torch

from sparse_key_value_b200.inputs import WORKLOADS, decode_step_inputs, make_inputs


def _selected_rows(w):
    """Rows the product-key lookup selects (fp32 torch on the CPU; a
    statistic of the inputs, not a parity reference)."""
    inp = make_inputs(w, "cpu", with_values=False)
    q, K = inp["query"].float(), inp["subkeys"].float()
    T, H = q.shape[:2]
    n, k = K.shape[2], w.k
    u = q / q.norm(dim=-1, keepdim=True)
    kap = K / K.norm(dim=-1, keepdim=True)
    out = []
    for h in range(H):
        v1, a1 = (u[:, h, 0] @ kap[h, 0].T).topk(k, dim=-1)
        v2, a2 = (u[:, h, 1] @ kap[h, 1].T).topk(k, dim=-1)
        top = (v1[:, :, None] + v2[:, None, :]).view(T, -1).topk(k, dim=-1).indices
        out.append(torch.gather(a1, 1, top // k) * n + torch.gather(a2, 1, top % k))
    return torch.cat(out).view(-1)


def test_train_workload_follows_zipf_1_1():
    torch.set_num_threads(max(1, torch.get_num_threads()))
    w = WORKLOADS["train"]
    ids = _selected_rows(w)
    cnt = torch.bincount(ids, minlength=w.N).double()
    c = torch.sort(cnt, descending=True).values[:10000].clamp_min(0.5)
    r = torch.arange(1, 10001, dtype=torch.float64)
    X = torch.stack([torch.ones_like(r), r.log()], 1)
    slope = torch.linalg.lstsq(X, c.log().unsqueeze(1)).solution[1, 0].item()
    assert -slope == pytest.approx(1.1, abs=0.05)
    assert 5e4 < int((cnt > 0).sum()) < 5e5


def test_workload_shapes():
    assert WORKLOADS["pkm"].N == 1 << 20
    assert WORKLOADS["memplus"].N == 1 << 24
    assert WORKLOADS["pkm"].N * WORKLOADS["pkm"].d_v * 2 == 4 << 30
    assert WORKLOADS["memplus"].N * WORKLOADS["memplus"].d_v * 2 == 32 << 30
    t = WORKLOADS["tiny"]
    assert (t.T, t.H, t.d_half, t.n_sub, t.k, t.d_v, t.dtype, t.seed) == \
        (512, 1, 128, 32, 8, 256, "f32", 0)


def test_decode_reuses_memplus_tables():
    m, d = WORKLOADS["memplus"], WORKLOADS["decode"]
    a = make_inputs(m.scaled(T=4), "cpu", with_values=False)
    b = make_inputs(d.scaled(T=8), "cpu", with_values=False)
    assert torch.equal(a["subkeys"], b["subkeys"])
    assert torch.equal(a["W1"], b["W1"]) and torch.equal(a["W2"], b["W2"])
    s0, s1 = decode_step_inputs(d, 0), decode_step_inputs(d, 1)
    assert s0["query"].shape == (8, 4, 2, 512)
    assert not torch.equal(s0["query"], s1["query"])


def test_distributions():
    w = WORKLOADS["pkm"].scaled(T=512, n_sub=64, d_v=64)
    inp = make_inputs(w, "cpu")
    assert abs(inp["query"].float().std().item() - 1.0) < 0.02
    assert abs(inp["subkeys"].float().std().item() - 1 / math.sqrt(512)) < 0.002
    assert abs(inp["values"].float().std().item() - 0.02) < 0.001


def test_engram_workload_and_bytes():
    """The Engram workload's shape and the bench's algorithmic bytes per
    token: one d-row per head, the hidden-state and output rows, alpha and
    the token id."""
    import os
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from sparse_key_value_b200.inputs import ENGRAM, make_engram_inputs

    w = ENGRAM
    assert (w.T, w.heads, w.d) == (16384, 8, 1024)
    assert len(set(w.seeds)) == w.heads and all(0 <= x < 2 ** 64 for x in w.seeds)
    assert w.n_rows == sum(w.rows_per_head) < 2 ** 31
    assert bench.engram_bytes_per_token(w) == 8 * 1024 * 2 + 2 * 1024 * 2 + 8
    small = w.scaled(n_seq=2, L=5, rows_per_head=(11,) * 8, d=16)
    inp = make_engram_inputs(small, "cpu")
    assert inp["tokens"].shape == (2, 5) and inp["tokens"].dtype == torch.int32
    assert inp["table"].shape == (88, 16) and inp["h"].shape == (10, 16)
    assert int(inp["tokens"].min()) >= 0 and int(inp["tokens"].max()) < small.vocab
    # the tables and hash seeds depend on the table seed only, the tokens on the seed
    other = make_engram_inputs(small.scaled(seed=small.seed + 1), "cpu")
    assert torch.equal(other["table"], inp["table"]) and not torch.equal(other["tokens"],
                                                                          inp["tokens"])
    assert small.scaled(seed=small.seed + 1).seeds == small.seeds


def test_traffic_records_follow_their_sources(tmp_path, monkeypatch):
    """bench.py reports an ncu traffic record only while every kernel source
    it names is unchanged (by hash); multi-source records need all of them."""
    import hashlib
    import json
    import os
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench

    def sha(name):
        path = os.path.join(root, "sparse_key_value_b200", "csrc", name)
        return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]

    rec = {
        "a": {"source": "k_embbag.cu", "source_sha": sha("k_embbag.cu"),
              "dram_bytes_per_launch": 11},
        "b": {"source": "k_embbag.cu", "source_sha": "0" * 16, "dram_bytes_per_launch": 12},
        "c:backward": {"sources": {"k_segsum.cu": sha("k_segsum.cu"),
                                   "k_sort.cu": sha("k_sort.cu")},
                       "dram_bytes_per_launch": 13, "l2_bytes_per_launch": 14},
        "d:backward": {"sources": {"k_segsum.cu": sha("k_segsum.cu"), "k_sort.cu": "1" * 16},
                       "dram_bytes_per_launch": 15, "l2_bytes_per_launch": 16},
    }
    (tmp_path / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.traffic_record("a") == 11
    assert bench.traffic_record("b") is None          # its kernel changed since the capture
    assert bench.traffic_record("missing") is None
    assert bench.traffic_entry("c:backward")["l2_bytes_per_launch"] == 14
    assert bench.traffic_entry("d:backward") is None  # one of its sources changed
