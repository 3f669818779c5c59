"""The device failure path without a GPU fault: a bounded wait that runs
out records PKM_ERR_TIMEOUT, the kernel returns, the status is read and
cleared on the host, and the context keeps working."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

skv = pytest.importorskip("sparse_key_value_b200")
from sparse_key_value_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    skv.load()
    assert skv.device_error() == 0
    yield


@pytest.mark.parametrize("polls", [1, 256, 4096])
def test_wait_runs_out_and_reports(polls):
    assert skv.check_wait_timeout(polls) == 5  # PKM_ERR_TIMEOUT
    assert skv.device_error() == 0             # read and cleared


def test_context_usable_after_a_timeout():
    assert skv.check_wait_timeout(1024) == 5
    w = WORKLOADS["pkm"].scaled(T=130, H=2, d_half=128, n_sub=256, k=8, d_v=64, seed=3)
    inp = make_inputs(w, "cuda")
    a = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    b = skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert np.isfinite(a[0].float().cpu().numpy()).all()
