"""Product-key memory lookup on B200 (sm_100a): torch-facing binding of
libpkm.so.

Every function here marshals torch tensors into the C ABI declared in
include/pkm.h and calls it on the current CUDA stream; the computation runs
entirely in the library's kernels.  Outputs and workspaces the caller does
not pass are allocated with torch (device memory only); the library itself
never allocates.
"""

from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._lib import (PKM_BF16, PKM_F32, PKMError, BwdArgs, FwdArgs, check, load)

__all__ = ["PKMError", "load", "pkm_forward", "pkm_backward", "embbag_forward",
           "embbag_backward", "forward_workspace_size", "backward_workspace_size",
           "device_error", "fwd_args"]


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PKM_BF16
    if t.dtype == torch.float32:
        return PKM_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _stream(dev: torch.device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libpkm works on CUDA tensors only")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def fwd_args(T, H, d_half, n_sub, k, d_v, dtype=PKM_BF16, d_model=0, memplus=False,
             **ptrs) -> FwdArgs:
    a = FwdArgs()
    a.T, a.H, a.d_half, a.n_sub, a.k, a.d_v, a.dtype = T, H, d_half, n_sub, k, d_v, dtype
    a.d_model = d_model
    if memplus:  # the size query only needs to know Memory+ is on
        a.x = a.W1 = a.W2 = ctypes.c_void_p(16)
    for name, v in ptrs.items():
        setattr(a, name, v)
    return a


def forward_workspace_size(T, H, d_half, n_sub, k, d_v, dtype=PKM_BF16, memplus=False,
                           d_model=0) -> int:
    a = fwd_args(T, H, d_half, n_sub, k, d_v, dtype, d_model, memplus)
    return int(load().pkm_forward_workspace_size(ctypes.byref(a)))


def pkm_forward(query, subkeys, values, k: int, x=None, W1=None, W2=None, out=None, idx=None,
                weights=None, workspace=None, stream=None, phase_events=None, y_out=None):
    """Forward of one memory layer (see pkm_forward in include/pkm.h).

    query [T,H,2,d_half], subkeys [H,2,n_sub,d_half], values [n_sub^2, d_v];
    optional Memory+ gate x [T,d_model], W1 [d_model,d_v], W2 [d_v,d_model].
    ``phase_events``: optional list of 7 torch.cuda.Event recorded at the
    phase boundaries (see pkm_fwd_args.phase_events).
    ``y_out``: Memory+ only, a [T, d_v] tensor receiving the bag output
    before the gate (what memplus_backward needs).
    Returns (out, idx, weights)."""
    _need_cuda(query, subkeys, values, x, W1, W2)
    T, H, two, dh = query.shape
    n = subkeys.shape[2]
    dv = values.shape[1]
    dev = query.device
    memplus = x is not None
    dm = x.shape[1] if memplus else 0
    if out is None:
        out = torch.empty(T, dm if memplus else dv, dtype=query.dtype, device=dev)
    if idx is None:
        idx = torch.empty(T, H, k, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(T, H, k, dtype=torch.float32, device=dev)
    a = fwd_args(T, H, dh, n, k, dv, _dt(query), dm, False, query=_p(query), subkeys=_p(subkeys),
                 values=_p(values), x=_p(x), W1=_p(W1), W2=_p(W2), out=_p(out), idx=_p(idx),
                 weights=_p(weights))
    lib = load()
    need = int(lib.pkm_forward_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _p(workspace), workspace.numel()
    a.y_out = _p(y_out)
    if phase_events is not None:
        if len(phase_events) != 7 or any(e.cuda_event == 0 for e in phase_events):
            raise ValueError("phase_events: 7 events, each recorded once before use")
        arr = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
        a.phase_events = ctypes.cast(arr, ctypes.c_void_p)
    check(lib.pkm_forward(ctypes.byref(a), _stream(dev, stream)), "pkm_forward")
    return out, idx, weights


def _bwd_args(query, subkeys, values, idx, weights, dy, **kw) -> BwdArgs:
    T, H, _, dh = query.shape
    a = BwdArgs()
    a.T, a.H, a.d_half, a.n_sub, a.k, a.d_v = T, H, dh, subkeys.shape[2], idx.shape[2], \
        values.shape[1]
    a.dtype = _dt(query)
    a.query, a.subkeys, a.values = _p(query), _p(subkeys), _p(values)
    a.idx, a.weights, a.dy = _p(idx), _p(weights), _p(dy)
    for name, v in kw.items():
        setattr(a, name, v)
    return a


def backward_workspace_size(query, subkeys, values, idx, weights, dy) -> int:
    a = _bwd_args(query, subkeys, values, idx, weights, dy)
    return int(load().pkm_backward_workspace_size(ctypes.byref(a)))


def pkm_backward(query, subkeys, values, idx, weights, dy, sparse: bool = True,
                 dense: Optional[torch.Tensor] = None, want_dscores: bool = False,
                 workspace=None, stream=None, uniq_cap: Optional[int] = None):
    """Backward of the plain lookup (see pkm_backward in include/pkm.h).

    Returns dict(dquery, dsubkeys, uniq_rows, grad_rows, n_uniq, dscores)
    with the sparse value gradient sliced to its n_uniq rows (a host read of
    n_uniq) when ``sparse``; ``dense`` [N, d_v] fp32 receives += if given."""
    _need_cuda(query, subkeys, values, idx, weights, dy, dense)
    T, H, _, dh = query.shape
    dev = query.device
    k = idx.shape[2]
    R = T * H * k
    dq = torch.empty(T, H, 2, dh, dtype=torch.float32, device=dev)
    dK = torch.empty_like(subkeys, dtype=torch.float32)
    cap = R if uniq_cap is None else uniq_cap
    uniq = torch.empty(max(cap, 1), dtype=torch.int32, device=dev) if sparse else None
    grad = torch.empty(max(cap, 1), values.shape[1], dtype=torch.float32, device=dev) \
        if sparse else None
    n_uniq = torch.zeros(1, dtype=torch.int64, device=dev) if sparse else None
    dS = torch.empty(T, H, k, dtype=torch.float32, device=dev) if want_dscores else None
    a = _bwd_args(query, subkeys, values, idx, weights, dy, dquery=_p(dq), dsubkeys=_p(dK),
                  uniq_rows=_p(uniq), grad_rows=_p(grad), n_uniq=_p(n_uniq),
                  uniq_cap=cap if sparse else 0, dvalues_dense=_p(dense), dscores=_p(dS))
    lib = load()
    need = int(lib.pkm_backward_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _p(workspace), workspace.numel()
    check(lib.pkm_backward(ctypes.byref(a), _stream(dev, stream)), "pkm_backward")
    res = dict(dquery=dq, dsubkeys=dK, dscores=dS, n_uniq=n_uniq)
    if sparse:
        u = int(n_uniq.item())
        res.update(uniq_rows=uniq[:u], grad_rows=grad[:u])
    return res


def embbag_forward(table, idx, w, gate=None, out=None, stream=None):
    """out[t] = (sum_j w[t,j] table[idx[t,j]]) (⊙ gate[t]); idx int32, w fp32 [n_bags, B]."""
    _need_cuda(table, idx, w, gate)
    n_bags, B = idx.shape
    d = table.shape[1]
    if out is None:
        out = torch.empty(n_bags, d, dtype=table.dtype, device=table.device)
    check(load().embbag_forward(_p(table), table.shape[0], d, _dt(table), _p(idx), _p(w),
                                n_bags, B, _p(gate), _p(out), _stream(table.device, stream)),
          "embbag_forward")
    return out


def embbag_backward(dy, idx, w, table=None, n_rows=None, sparse=True, dense=None,
                    want_dw=False, stream=None):
    """Backward of embbag_forward (no gate); see include/pkm.h."""
    _need_cuda(dy, idx, w, table, dense)
    n_bags, B = idx.shape
    d = dy.shape[1]
    dev = dy.device
    n_rows = table.shape[0] if n_rows is None else n_rows
    R = n_bags * B
    dw = torch.empty(n_bags, B, dtype=torch.float32, device=dev) if want_dw else None
    uniq = torch.empty(max(R, 1), dtype=torch.int32, device=dev) if sparse else None
    grad = torch.empty(max(R, 1), d, dtype=torch.float32, device=dev) if sparse else None
    n_uniq = torch.zeros(1, dtype=torch.int64, device=dev) if sparse else None
    lib = load()
    need = int(lib.embbag_backward_workspace_size(n_bags, B, d, n_rows))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    check(lib.embbag_backward(_p(dy), _p(idx), _p(w), n_bags, B, d, _dt(dy), _p(table), n_rows,
                              _p(dw), _p(uniq), _p(grad), _p(n_uniq), R if sparse else 0,
                              _p(dense), _p(ws), ws.numel(), _stream(dev, stream)),
          "embbag_backward")
    res = dict(dw=dw)
    if sparse:
        u = int(n_uniq.item())
        res.update(uniq_rows=uniq[:u], grad_rows=grad[:u])
    return res


def device_error(stream=None, device=None) -> int:
    """Synchronise and read-and-clear the device status word (0 = none)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    code = ctypes.c_int32(0)
    check(load().pkm_get_device_error(_stream(dev, stream), ctypes.byref(code)),
          "pkm_get_device_error")
    return int(code.value)


def memplus_backward(x, W1, W2, y, dout, workspace=None, stream=None):
    """Backward of the Memory+ block (see pkm_memplus_backward in include/pkm.h).

    x [T,d_model], W1 [d_model,d_v], W2 [d_v,d_model], y [T,d_v] (the
    forward's y_out), dout [T,d_model], all bf16.  Returns dict(dy (bf16,
    the dy of pkm_backward), dx, dW1, dW2 (fp32))."""
    _need_cuda(x, W1, W2, y, dout)
    T, dm = x.shape
    dv = W1.shape[1]
    dev = x.device
    dy = torch.empty(T, dv, dtype=x.dtype, device=dev)
    dx = torch.empty(T, dm, dtype=torch.float32, device=dev)
    dW1 = torch.empty(dm, dv, dtype=torch.float32, device=dev)
    dW2 = torch.empty(dv, dm, dtype=torch.float32, device=dev)
    a = _lib.MemplusBwdArgs(T, dm, dv, _p(x), _p(W1), _p(W2), _p(y), _p(dout), _p(dy), _p(dx),
                            _p(dW1), _p(dW2), None, 0)
    lib = load()
    need = int(lib.pkm_memplus_backward_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _p(workspace), workspace.numel()
    check(lib.pkm_memplus_backward(ctypes.byref(a), _stream(dev, stream)), "pkm_memplus_backward")
    return dict(dy=dy, dx=dx, dW1=dW1, dW2=dW2)


def _qproj_args(x, Wq, q=None, dq=None, dWq=None, dx=None) -> "_lib.QprojArgs":
    T, dm = x.shape
    return _lib.QprojArgs(T, dm, Wq.shape[1], _p(x), _p(Wq), _p(q), _p(dq), _p(dWq), _p(dx),
                          None, 0)


def _qproj_call(fn: str, a, dev, workspace, stream):
    lib = load()
    need = int(lib.pkm_qproj_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _p(workspace), workspace.numel()
    check(getattr(lib, fn)(ctypes.byref(a), _stream(dev, stream)), fn)


def qproj_forward(x, Wq, out=None, workspace=None, stream=None):
    """q = x Wq (bf16 [T, d_q]; see pkm_qproj_forward in include/pkm.h)."""
    _need_cuda(x, Wq)
    if out is None:
        out = torch.empty(x.shape[0], Wq.shape[1], dtype=x.dtype, device=x.device)
    _qproj_call("pkm_qproj_forward", _qproj_args(x, Wq, q=out), x.device, workspace, stream)
    return out


def qproj_backward(x, Wq, dq, dx=None, workspace=None, stream=None):
    """dWq = x^T dq and dx += dq Wq^T (dq fp32 [T, d_q]; dx fp32 [T, d_model],
    zero-initialised when not given).  Returns dict(dWq, dx)."""
    _need_cuda(x, Wq, dq)
    dev = x.device
    if dx is None:
        dx = torch.zeros(x.shape[0], x.shape[1], dtype=torch.float32, device=dev)
    dWq = torch.empty(x.shape[1], Wq.shape[1], dtype=torch.float32, device=dev)
    dq = dq.reshape(x.shape[0], Wq.shape[1]).contiguous()
    _qproj_call("pkm_qproj_backward", _qproj_args(x, Wq, dq=dq, dWq=dWq, dx=dx), dev, workspace,
                stream)
    return dict(dWq=dWq, dx=dx)


def sparse_optimizer_step(table, rows, grads, count, lr: float, kind: str = "sgd", m=None,
                          v=None, betas=(0.9, 0.999), eps: float = 1e-8, step: int = 1,
                          stream=None):
    """In-place SGD or touched-rows Adam on the rows of a sparse value
    gradient (see pkm_sparse_optimizer_step in include/pkm.h): table
    [n_rows, d], rows int32 [cap], grads fp32 [cap, d], count device int64
    [1] (pkm_backward's uniq_rows, grad_rows, n_uniq); m, v fp32 [n_rows, d]
    for Adam."""
    _need_cuda(table, rows, grads, count, m, v)
    adam = kind == "adam"
    if adam and (m is None or v is None):
        raise ValueError("adam needs the moment tensors m and v")
    a = _lib.SparseOptArgs(1 if adam else 0, lr, betas[0], betas[1], eps, step, table.shape[0],
                           table.shape[1], _dt(table), _p(table), _p(rows), _p(grads), _p(count),
                           rows.shape[0], _p(m), _p(v))
    check(load().pkm_sparse_optimizer_step(ctypes.byref(a), _stream(table.device, stream)),
          "pkm_sparse_optimizer_step")
    return table


def engram_forward(tokens, table, h, orders, K: int, seeds, rows_per_head, alpha=True,
                   rows=False, e=False, out=None, stream=None):
    """Engram lookup (see pkm_engram_forward in include/pkm.h): hashed
    n-gram rows of the stacked table, their sum e and the context gate.

    tokens [n_seq, L] int32, table [sum(rows_per_head), d], h [T, d] CUDA
    tensors (T = n_seq * L); orders, seeds and rows_per_head host sequences
    (head j = o*K + k).  Returns dict(v, alpha, rows, e), the optional ones
    None unless asked for."""
    _need_cuda(tokens, table, h, out)
    if tokens.dtype != torch.int32:
        raise TypeError("tokens must be int32")
    n_seq, L = tokens.shape
    T, d = h.shape
    if T != n_seq * L or table.shape[1] != d or table.dtype != h.dtype:
        raise ValueError("shapes: tokens [n_seq, L], h [n_seq*L, d], table [rows, d], one dtype")
    dev = h.device
    heads = len(orders) * K
    od = (ctypes.c_int32 * len(orders))(*orders)
    sd = (ctypes.c_uint64 * heads)(*[int(x) & (2 ** 64 - 1) for x in seeds])
    md = (ctypes.c_int64 * heads)(*rows_per_head)
    v = torch.empty(T, d, dtype=h.dtype, device=dev) if out is None else out
    a_t = torch.empty(T, dtype=torch.float32, device=dev) if alpha else None
    r_t = torch.empty(T, heads, dtype=torch.int32, device=dev) if rows else None
    e_t = torch.empty(T, d, dtype=h.dtype, device=dev) if e else None
    args = _lib.EngramArgs(n_seq, L, len(orders), K, ctypes.cast(od, ctypes.c_void_p),
                           ctypes.cast(sd, ctypes.c_void_p), ctypes.cast(md, ctypes.c_void_p),
                           d, _dt(h), _p(tokens), _p(table), _p(h), _p(v), _p(a_t), _p(r_t),
                           _p(e_t))
    check(load().pkm_engram_forward(ctypes.byref(args), _stream(dev, stream)),
          "pkm_engram_forward")
    return dict(v=v, alpha=a_t, rows=r_t, e=e_t)


def pkm_select(query, subkeys, k: int, d_v: int = 8, idx=None, weights=None, workspace=None,
               stream=None):
    """The selection alone (see pkm_select in include/pkm.h): returns (idx,
    weights) [T, H, k] as pkm_forward would."""
    _need_cuda(query, subkeys)
    T, H, two, dh = query.shape
    n = subkeys.shape[2]
    dev = query.device
    if idx is None:
        idx = torch.empty(T, H, k, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(T, H, k, dtype=torch.float32, device=dev)
    a = fwd_args(T, H, dh, n, k, d_v, _dt(query), 0, False, query=_p(query),
                 subkeys=_p(subkeys), idx=_p(idx), weights=_p(weights))
    lib = load()
    need = int(lib.pkm_forward_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = _p(workspace), workspace.numel()
    check(lib.pkm_select(ctypes.byref(a), _stream(dev, stream)), "pkm_select")
    return idx, weights


def embbag_forward_range(table_shard, row_lo: int, idx, w, out=None, stream=None):
    """Partial bags over one row shard (see embbag_forward_range in
    include/pkm.h): table_shard holds rows [row_lo, row_lo + len) of the full
    table; idx int32 / w fp32 [n_bags, B] hold full-table ids; returns fp32
    [n_bags, d]."""
    _need_cuda(table_shard, idx, w, out)
    n_bags, B = idx.shape
    d = table_shard.shape[1]
    if out is None:
        out = torch.empty(n_bags, d, dtype=torch.float32, device=table_shard.device)
    check(load().embbag_forward_range(_p(table_shard), row_lo, table_shard.shape[0], d,
                                      _dt(table_shard), _p(idx), _p(w), n_bags, B, _p(out),
                                      _stream(table_shard.device, stream)),
          "embbag_forward_range")
    return out


def check_wait_timeout(polls: int = 4096, device=None, stream=None) -> int:
    """Run the bounded-wait failure path (see pkm_check_wait_timeout in
    include/pkm.h) and return the device status it left (PKM_ERR_TIMEOUT = 5
    expected), after checking that the waiting kernel returned."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    done = torch.zeros(1, dtype=torch.int32, device=dev)
    check(load().pkm_check_wait_timeout(polls, _p(done), _stream(dev, stream)),
          "pkm_check_wait_timeout")
    code = device_error(stream, dev)
    if int(done.item()) != 1:
        raise RuntimeError(f"the waiting kernel did not finish as expected ({int(done.item())})")
    return code
