"""GPU parity of the Memory+ backward and the query projection against the
CPU oracle (through the C ABI).

"Memory Layers at Scale" digest, "Memory+ 블록": out = (y ⊙ silu(x W1)) W2;
the backward gives the gradient of the bag output (dy, which feeds the
lookup's backward), dx, dW1 and dW2.  The query projection q = x Wq feeds
the lookup from the layer input.  Operands are bf16 and the GEMMs round
their bf16 operands (dout, the gate product, da), so every fp32 output is
held to the bf16 rule: |gpu - ref| <= rtol (|ref| + RMS(ref)), rtol 2e-2.
"""

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


def _bf16(g, *shape, std=1.0):
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)


def _memplus_case(seed, T, dm, dv):
    g = torch.Generator().manual_seed(seed)
    x = _bf16(g, T, dm)
    W1 = _bf16(g, dm, dv, std=dm ** -0.5)
    W2 = _bf16(g, dv, dm, std=dv ** -0.5)
    y = _bf16(g, T, dv, std=0.1)
    dout = _bf16(g, T, dm)
    return x, W1, W2, y, dout


# (T, d_model, d_v): tensor-core GEMMs with a ragged token count; d_model = 32
# puts the K = d_model products on the SIMT GEMM; T < 64 pads the token axis;
# T = 4096 splits the token-contracting weight-gradient GEMMs over K
SHAPES = [(300, 256, 128), (130, 32, 48), (40, 64, 64), (1, 16, 8), (4096, 256, 256)]


@pytest.mark.parametrize("T,dm,dv", SHAPES, ids=[f"T{s[0]}-dm{s[1]}-dv{s[2]}" for s in SHAPES])
def test_memplus_backward_matches_oracle(T, dm, dv):
    import oracle

    x, W1, W2, y, dout = _memplus_case(1000 + T + dm + dv, T, dm, dv)
    r = skv.memplus_backward(x.cuda(), W1.cuda(), W2.cuda(), y.cuda(), dout.cuda())
    torch.cuda.synchronize()
    ref = oracle.memplus_backward(y.double().numpy(), x, W1, W2, dout)
    close(r["dy"].float().cpu().numpy(), ref["dy"], RTOL["bf16"], "dy")
    close(r["dx"].cpu().numpy(), ref["dx"], RTOL["bf16"], "dx")
    close(r["dW1"].cpu().numpy(), ref["dW1"], RTOL["bf16"], "dW1")
    close(r["dW2"].cpu().numpy(), ref["dW2"], RTOL["bf16"], "dW2")


def test_memplus_backward_deterministic():
    x, W1, W2, y, dout = (t.cuda() for t in _memplus_case(7, 257, 128, 64))
    a = skv.memplus_backward(x, W1, W2, y, dout)
    b = skv.memplus_backward(x, W1, W2, y, dout)
    torch.cuda.synchronize()
    for key in a:
        assert torch.equal(a[key], b[key]), key


# (T, d_model, d_q): more than 128 tokens runs the GEMMs on SM pairs (256-row
# tiles, a ragged last pair); 50 tokens the single-SM tensor-core kernel;
# 4100 x 1024 x 1024 many tiles per pair with a ragged tail
QPROJ = [(300, 128, 256), (50, 32, 64), (1000, 640, 520), (4100, 1024, 1024)]


@pytest.mark.parametrize("T,dm,dq", QPROJ)
def test_qproj_matches_oracle(T, dm, dq):
    import oracle

    g = torch.Generator().manual_seed(T + dm + dq)
    x, Wq = _bf16(g, T, dm), _bf16(g, dm, dq, std=dm ** -0.5)
    dq_in = torch.randn(T, dq, generator=g)
    q = skv.qproj_forward(x.cuda(), Wq.cuda())
    dx0 = torch.randn(T, dm, generator=g)
    r = skv.qproj_backward(x.cuda(), Wq.cuda(), dq_in.cuda(), dx=dx0.clone().cuda())
    torch.cuda.synchronize()
    close(q.float().cpu().numpy(), oracle.qproj(x, Wq), RTOL["bf16"], "q")
    ref = oracle.qproj_backward(x, Wq, dq_in.double().numpy())
    close(r["dWq"].cpu().numpy(), ref["dWq"], RTOL["bf16"], "dWq")
    close(r["dx"].cpu().numpy(), ref["dx"] + dx0.double().numpy(), RTOL["bf16"], "dx (accumulated)")


def test_memplus_training_chain():
    """q = x Wq -> Memory+ forward keeping y -> Memory+ backward -> lookup
    backward -> query projection backward, each stage against the oracle on
    the GPU's own inputs to that stage; the forward with y_out agrees with
    the fused forward."""
    import oracle

    w = WORKLOADS["memplus"].scaled(name="mp-chain", T=256, H=2, d_half=256, n_sub=256, k=16,
                                    d_v=128, d_model=128, train=True)
    inp = make_inputs(w, "cuda")
    g = torch.Generator().manual_seed(31)
    dq_total = w.H * 2 * w.d_half
    Wq = _bf16(g, w.d_model, dq_total, std=w.d_model ** -0.5).cuda()
    x, W1, W2 = inp["x"], inp["W1"], inp["W2"]
    q = skv.qproj_forward(x, Wq).view(w.T, w.H, 2, w.d_half)
    y = torch.empty(w.T, w.d_v, dtype=torch.bfloat16, device="cuda")
    out, idx, wts = skv.pkm_forward(q, inp["subkeys"], inp["values"], w.k, x=x, W1=W1, W2=W2,
                                    y_out=y)
    out_fused, idx_f, _ = skv.pkm_forward(q, inp["subkeys"], inp["values"], w.k, x=x, W1=W1,
                                          W2=W2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_f)
    close(out.float().cpu().numpy(), out_fused.double().cpu().numpy(), RTOL["bf16"], "out")
    # y is the plain bag of the selection
    rows = np.unique(idx.cpu().numpy().astype(np.int64))
    V = inp["values"][torch.from_numpy(rows).cuda()].cpu()
    vrow = np.searchsorted(rows, idx.cpu().numpy().astype(np.int64))
    y_ref = oracle.bag(vrow.reshape(w.T, -1), wts.double().cpu().numpy().reshape(w.T, -1), V)
    close(y.float().cpu().numpy(), y_ref, RTOL["bf16"], "y")
    # Memory+ backward
    dout = _bf16(g, w.T, w.d_model).cuda()
    mp = skv.memplus_backward(x, W1, W2, y, dout)
    ref = oracle.memplus_backward(y.double().cpu().numpy(), x.cpu(), W1.cpu(), W2.cpu(),
                                  dout.cpu())
    for key in ("dy", "dx", "dW1", "dW2"):
        close(mp[key].float().cpu().numpy(), ref[key], RTOL["bf16"], key)
    # lookup backward on the Memory+ dy, then the projection's backward
    gr = skv.pkm_backward(q, inp["subkeys"], inp["values"], idx, wts, mp["dy"])
    qp = skv.qproj_backward(x, Wq, gr["dquery"].view(w.T, -1), dx=mp["dx"].clone())
    torch.cuda.synchronize()
    ref_q = oracle.qproj_backward(x.cpu(), Wq.cpu(), gr["dquery"].double().cpu().numpy()
                                  .reshape(w.T, -1))
    close(qp["dWq"].cpu().numpy(), ref_q["dWq"], RTOL["bf16"], "dWq")
    close(qp["dx"].cpu().numpy(), ref_q["dx"] + mp["dx"].double().cpu().numpy(), RTOL["bf16"],
          "dx (Memory+ and projection)")
