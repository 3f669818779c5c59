"""The allocation-free forward entry point, through the C ABI.

Some callers cannot allocate device memory for the forward's scratch: a C
program that links only libpkm.so and has no allocator of its own, a serving
runtime whose device memory budget is fixed at start-up, or a latency-critical
loop that must not call the synchronising cudaMalloc.  pkm_forward_noalloc
serves them with a fixed scratch array inside the library.  These tests check
it against pkm_forward on two calls in a row (the array keeps the previous
call's contents, so the second call must not depend on them) and check that a
request beyond the array is refused.  The file runs last so that a failure
here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

from parity import RTOL

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def _call_noalloc(inp, k):
    """Marshal the arguments like pkm_forward and call the C entry point."""
    q, K, V = inp["query"], inp["subkeys"], inp["values"]
    T, H, _, dh = q.shape
    mp = "x" in inp
    d_out = inp["W2"].shape[1] if mp else V.shape[1]
    out = torch.empty(T, d_out, dtype=q.dtype, device=q.device)
    idx = torch.empty(T, H, k, dtype=torch.int32, device=q.device)
    w = torch.empty(T, H, k, dtype=torch.float32, device=q.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    extra = dict(x=p(inp["x"]), W1=p(inp["W1"]), W2=p(inp["W2"])) if mp else {}
    a = skv.fwd_args(T, H, dh, K.shape[2], k, V.shape[1], 1 if q.dtype == torch.bfloat16 else 0,
                     d_model=d_out if mp else 0, query=p(q), subkeys=p(K), values=p(V),
                     out=p(out), idx=p(idx), weights=p(w), **extra)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = skv.load().pkm_forward_noalloc(ctypes.byref(a), stream)
    return rc, out, idx, w


def _check_same(inp, w, dt):
    """pkm_forward_noalloc against pkm_forward on the same inputs: equal row
    ids and weights, outputs within the dtype's tolerance."""
    rc, out, idx, wts = _call_noalloc(inp, w.k)
    assert rc == 0
    mp = "x" in inp
    ref_out, ref_idx, ref_w = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k,
                                              x=inp.get("x"), W1=inp.get("W1"),
                                              W2=inp.get("W2"))
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    assert torch.equal(idx, ref_idx)
    np.testing.assert_allclose(wts.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-6, atol=0)
    a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(b * b)))
    assert np.all(np.abs(a - b) <= RTOL[dt] * (np.abs(b) + rms)), mp


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    yield


def test_noalloc_matches_pkm_forward_two_calls():
    base = WORKLOADS["pkm"].scaled(T=1000, H=4, d_half=512, n_sub=1024, k=32, d_v=256)
    for seed in (11, 12):  # two calls in a row, different inputs
        w = base.scaled(seed=seed, table_seed_=seed + 100)
        inp = make_inputs(w, "cuda")
        rc, out, idx, wts = _call_noalloc(inp, w.k)
        assert rc == 0
        ref_out, ref_idx, ref_w = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"],
                                                  w.k)
        torch.cuda.synchronize()
        assert skv.device_error() == 0
        assert torch.equal(idx, ref_idx)
        np.testing.assert_allclose(wts.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-6, atol=0)
        a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
        rms = float(np.sqrt(np.mean(b * b)))
        assert np.all(np.abs(a - b) <= RTOL["bf16"] * (np.abs(b) + rms))


def test_noalloc_other_paths_after_a_large_call():
    """After a large call has filled the array: a decode-sized batch (column
    splits, the second combine kernel and the row-group partial sums of the
    small-batch gather all live in the array), an fp32 batch (SIMT scoring,
    its query norms and per-half lists in the array) and a Memory+ batch
    (transposed weights, gate and gated rows in the array), each against
    pkm_forward."""
    big = WORKLOADS["pkm"].scaled(T=1000, H=4, d_half=512, n_sub=1024, k=32, d_v=256, seed=21)
    _check_same(make_inputs(big, "cuda"), big, "bf16")
    small = WORKLOADS["pkm"].scaled(T=8, H=4, d_half=512, n_sub=1024, k=32, d_v=256, seed=22)
    _check_same(make_inputs(small, "cuda"), small, "bf16")
    f32 = WORKLOADS["tiny"].scaled(T=100, seed=23)
    _check_same(make_inputs(f32, "cuda"), f32, "f32")
    mp = WORKLOADS["memplus"].scaled(T=200, H=2, d_half=64, n_sub=256, k=16, d_v=256,
                                     d_model=128, seed=24, table_seed_=25)
    _check_same(make_inputs(mp, "cuda"), mp, "bf16")


def test_noalloc_invalid_arguments_before_sizing():
    """Invalid sizes are refused as invalid (status 1), before any workspace
    size is computed from them, and launch nothing."""
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced
    lib = skv.load()
    for kw in (dict(k=0), dict(T=-5), dict(H=-1), dict(d_v=-8), dict(k=40, n_sub=16),
               dict(T=(1 << 36) + 1)):
        sizes = dict(T=64, H=4, d_half=512, n_sub=1024, k=32, d_v=256)
        sizes.update(kw)
        a = skv.fwd_args(sizes["T"], sizes["H"], sizes["d_half"], sizes["n_sub"], sizes["k"],
                         sizes["d_v"], 1, query=fake, subkeys=fake, values=fake, out=fake,
                         idx=fake, weights=fake)
        assert lib.pkm_forward_noalloc(ctypes.byref(a), None) == 1, kw


def test_noalloc_refuses_oversize_request():
    # fp32 scoring keeps per-half lists of every token in the scratch: 128 MiB here
    w = WORKLOADS["pkm"].scaled(T=65536, H=4, d_half=512, n_sub=1024, k=32, d_v=64)
    need = skv.forward_workspace_size(w.T, w.H, w.d_half, w.n_sub, w.k, w.d_v, 0)
    assert need > (32 << 20)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: refused before any launch
    a = skv.fwd_args(w.T, w.H, w.d_half, w.n_sub, w.k, w.d_v, 0, query=fake, subkeys=fake,
                     values=fake, out=fake, idx=fake, weights=fake)
    rc = skv.load().pkm_forward_noalloc(ctypes.byref(a), None)
    assert rc == 6  # PKM_ERR_WORKSPACE
