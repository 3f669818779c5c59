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
    out = torch.empty(T, V.shape[1], dtype=q.dtype, device=q.device)
    idx = torch.empty(T, H, k, dtype=torch.int32, device=q.device)
    w = torch.empty(T, H, k, dtype=torch.float32, device=q.device)
    a = skv.fwd_args(T, H, dh, K.shape[2], k, V.shape[1], 1 if q.dtype == torch.bfloat16 else 0,
                     query=ctypes.c_void_p(q.data_ptr()), subkeys=ctypes.c_void_p(K.data_ptr()),
                     values=ctypes.c_void_p(V.data_ptr()), out=ctypes.c_void_p(out.data_ptr()),
                     idx=ctypes.c_void_p(idx.data_ptr()), weights=ctypes.c_void_p(w.data_ptr()))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = skv.load().pkm_forward_noalloc(ctypes.byref(a), stream)
    return rc, out, idx, w


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


def test_noalloc_refuses_oversize_request():
    w = WORKLOADS["pkm"].scaled(T=65536, H=4, d_half=512, n_sub=1024, k=32, d_v=64)
    need = skv.forward_workspace_size(w.T, w.H, w.d_half, w.n_sub, w.k, w.d_v)
    assert need > (32 << 20)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: refused before any launch
    a = skv.fwd_args(w.T, w.H, w.d_half, w.n_sub, w.k, w.d_v, 1, query=fake, subkeys=fake,
                     values=fake, out=fake, idx=fake, weights=fake)
    rc = skv.load().pkm_forward_noalloc(ctypes.byref(a), None)
    assert rc == 6  # PKM_ERR_WORKSPACE
