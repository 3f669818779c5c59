"""CPU oracle for the product-key memory lookup (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python
binding never do: the two implementations share no code.

The arithmetic lives in ``pkm_oracle.c`` (plain C, IEEE double, OpenMP over
(token, head)); this module only compiles it and marshals numpy arrays.
Each function states which passage of the pages it follows:

* "Memory Layers at Scale" digest, "Product-key 검색": split keys, top-k
  from 2*sqrt(N) comparisons.
* "Memory Layers at Scale" digest, "Memory+ 블록": (y ⊙ silu(x W1)) W2 and
  qk-normalization.
* "Memory Layers at Scale" digest, "병렬 EmbeddingBag 구현": the weighted bag.
* "모델 안의 메모리", "작동 방식" and figure D: halves scored against the
  half-keys, best of each combined, weighted average of the values read.
* "Conditional Memory via Scalable Lookup" review (Engram), "희소 검색" and
  "핵심 수식": multi-head hashed n-gram rows, the context gate.

Parity pins (tests/test_oracle_pins.py) tie every function to something other
than itself: brute force over all N keys, closed forms, numpy/torch library
special cases and finite differences.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkm_oracle.c")
_HDR = os.path.join(_HERE, "pkm_oracle.h")
_LIB = os.path.join(_HERE, "liboracle_pkm.so")

F64, F32, BF16 = 0, 1, 2
NORM_EPS = 1e-12

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle_pkm.so`` (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64, I = ctypes.c_int64, ctypes.c_int
        lib.orc_half_scores.argtypes = [I64, I, I, I, P, I, P, I, P]
        lib.orc_topk.argtypes = [P, I, I, P]
        lib.orc_pkm_select.argtypes = [I64, I, I, I, I, P, I, P, I, P, P, P, P]
        lib.orc_bruteforce_select.argtypes = [I64, I, I, I, I, P, I, P, I, P, P]
        lib.orc_softmax.argtypes = [P, I64, I, P]
        lib.orc_bag.argtypes = [I64, I, I, P, P, P, I, I64, P]
        lib.orc_memplus.argtypes = [I64, I, I, P, P, I, P, I, P, I, P]
        lib.orc_pkm_backward.argtypes = [I64, I, I, I, I, I, P, I, P, I, P, I, I64,
                                         P, P, P, P, I, P, P, P, P, P]
        lib.orc_value_grad_rows.argtypes = [I64, I, I, I, P, P, P, I, P, I64, P]
        lib.orc_memplus_backward.argtypes = [I64, I, I, P, P, I, P, I, P, I, P, I, P, P, P, P]
        lib.orc_qproj.argtypes = [I64, I, I, P, I, P, I, P]
        lib.orc_qproj_backward.argtypes = [I64, I, I, P, I, P, I, P, P, P]
        lib.orc_engram_rows.argtypes = [I64, I, P, I, P, I, P, P, P]
        lib.orc_engram_gate.argtypes = [I64, I, I, P, P, I, I64, P, I, ctypes.c_double, P, P,
                                        P]
        lib.orc_num_threads.argtypes = []
        for f in ("orc_half_scores", "orc_topk", "orc_pkm_select",
                  "orc_bruteforce_select", "orc_softmax", "orc_bag", "orc_memplus",
                  "orc_pkm_backward", "orc_num_threads", "orc_value_grad_rows",
                  "orc_memplus_backward", "orc_qproj", "orc_qproj_backward",
                  "orc_engram_rows", "orc_engram_gate"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _input(x):
    """(contiguous numpy array, dtype tag) for a numpy array or torch tensor.

    bf16 tensors travel as their raw 16-bit patterns and are decoded exactly
    by the C code; fp32 and fp64 are passed as they are.
    """
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            return x.to(torch.float64).numpy(), F64
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return int(_load().orc_num_threads())


def half_scores(q, K):
    """s[t,h,c,a] = sqrt(dh) * <q_c/|q_c|, K_c[a]/|K_c[a]|>  (shape [T,H,2,n])."""
    qa, qt = _input(q)
    ka, kt = _input(K)
    T, H, two, dh = qa.shape
    n = ka.shape[2]
    out = np.empty((T, H, 2, n), np.float64)
    _check(_load().orc_half_scores(T, H, dh, n, _p(qa), qt, _p(ka), kt, _p(out)),
           "half_scores")
    return out


def topk(s, k: int):
    """Positions of the k largest entries of the 1-D array s, larger first,
    equal values -> smaller position first."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    pos = np.empty(k, np.int32)
    _check(_load().orc_topk(_p(s), s.shape[0], k, _p(pos)), "topk")
    return pos


def pkm_select(q, K, k: int):
    """Product-key selection.  Returns (idx int64 [T,H,k], S [T,H,k],
    w [T,H,k], number of half-key dot products evaluated)."""
    qa, qt = _input(q)
    ka, kt = _input(K)
    T, H, _, dh = qa.shape
    n = ka.shape[2]
    idx = np.empty((T, H, k), np.int64)
    S = np.empty((T, H, k), np.float64)
    w = np.empty((T, H, k), np.float64)
    dots = ctypes.c_int64(0)
    _check(_load().orc_pkm_select(T, H, dh, n, k, _p(qa), qt, _p(ka), kt, _p(idx),
                                  _p(S), _p(w), ctypes.byref(dots)), "pkm_select")
    return idx, S, w, int(dots.value)


def bruteforce_select(q, K, k: int):
    """Top-k over all N = n*n full keys.  Returns (idx [T,H,k], S [T,H,k])."""
    qa, qt = _input(q)
    ka, kt = _input(K)
    T, H, _, dh = qa.shape
    n = ka.shape[2]
    idx = np.empty((T, H, k), np.int64)
    S = np.empty((T, H, k), np.float64)
    _check(_load().orc_bruteforce_select(T, H, dh, n, k, _p(qa), qt, _p(ka), kt,
                                         _p(idx), _p(S)), "bruteforce_select")
    return idx, S


def softmax(S):
    S = np.ascontiguousarray(S, dtype=np.float64)
    k = S.shape[-1]
    w = np.empty_like(S)
    _check(_load().orc_softmax(_p(S), S.size // k, k, _p(w)), "softmax")
    return w


def bag(idx, w, table):
    """y[t] = sum_j w[t,j] * table[idx[t,j]]; idx/w [n_bags, B]."""
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    ta, tt = _input(table)
    n_bags = idx.shape[0]
    B = int(np.prod(idx.shape[1:]))
    d = ta.shape[1]
    y = np.empty((n_bags, d), np.float64)
    _check(_load().orc_bag(n_bags, B, d, _p(idx), _p(w), _p(ta), tt, ta.shape[0],
                           _p(y)), "bag")
    return y


def memplus(y, x, W1, W2):
    """out = (y ⊙ silu(x W1)) W2."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    xa, xt = _input(x)
    w1, w1t = _input(W1)
    w2, w2t = _input(W2)
    T, dm = xa.shape
    dv = w1.shape[1]
    out = np.empty((T, dm), np.float64)
    _check(_load().orc_memplus(T, dm, dv, _p(y), _p(xa), xt, _p(w1), w1t, _p(w2), w2t,
                               _p(out)), "memplus")
    return out


def memplus_backward(y, x, W1, W2, dout):
    """Backward of out = (y ⊙ silu(x W1)) W2 ("Memory+ 블록").

    Returns dict(dy [T,dv] (the gradient into the bag output), dx [T,dm],
    dW1 [dm,dv], dW2 [dv,dm]).
    """
    y = np.ascontiguousarray(y, dtype=np.float64)
    xa, xt = _input(x)
    w1, w1t = _input(W1)
    w2, w2t = _input(W2)
    da, dt = _input(dout)
    T, dm = xa.shape
    dv = w1.shape[1]
    dy = np.empty((T, dv))
    dx = np.empty((T, dm))
    dW1 = np.empty((dm, dv))
    dW2 = np.empty((dv, dm))
    _check(_load().orc_memplus_backward(T, dm, dv, _p(y), _p(xa), xt, _p(w1), w1t, _p(w2), w2t,
                                        _p(da), dt, _p(dy), _p(dx), _p(dW1), _p(dW2)),
           "memplus_backward")
    return dict(dy=dy, dx=dx, dW1=dW1, dW2=dW2)


def qproj(x, Wq):
    """q = x Wq: every head's and half's query from the layer input."""
    xa, xt = _input(x)
    wa, wt = _input(Wq)
    T, dm = xa.shape
    dq = wa.shape[1]
    q = np.empty((T, dq))
    _check(_load().orc_qproj(T, dm, dq, _p(xa), xt, _p(wa), wt, _p(q)), "qproj")
    return q


def qproj_backward(x, Wq, dq):
    """Backward of q = x Wq: dict(dWq [dm,dq], dx [T,dm])."""
    xa, xt = _input(x)
    wa, wt = _input(Wq)
    dq = np.ascontiguousarray(dq, dtype=np.float64)
    T, dm = xa.shape
    d_q = wa.shape[1]
    dWq = np.empty((dm, d_q))
    dx = np.empty((T, dm))
    _check(_load().orc_qproj_backward(T, dm, d_q, _p(xa), xt, _p(wa), wt, _p(dq), _p(dWq),
                                      _p(dx)), "qproj_backward")
    return dict(dWq=dWq, dx=dx)


def pkm_backward(q, K, table, idx, vrow, w, dy, want_dv: bool = True):
    """Backward of the lookup with the selection held fixed.

    ``idx`` [T,H,k] holds global row ids (a*n+b); ``vrow`` [T,H,k] the
    position of each selected row in the compact ``table`` [n_rows, d_v].
    Returns dict(dw, dS [T,H,k], dq [T,H,2,dh], dK [H,2,n,dh],
    dV [n_rows, d_v] or None).
    """
    qa, qt = _input(q)
    ka, kt = _input(K)
    ta, tt = _input(table)
    da, dt = _input(dy)
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    vrow = np.ascontiguousarray(vrow, dtype=np.int64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, H, _, dh = qa.shape
    n = ka.shape[2]
    k = idx.shape[-1]
    dv = ta.shape[1]
    dw = np.empty((T, H, k))
    dS = np.empty((T, H, k))
    dq = np.empty((T, H, 2, dh))
    dK = np.empty((H, 2, n, dh))
    dV = np.empty((ta.shape[0], dv)) if want_dv else None
    _check(_load().orc_pkm_backward(
        T, H, dh, n, k, dv, _p(qa), qt, _p(ka), kt, _p(ta), tt, ta.shape[0],
        _p(idx), _p(vrow), _p(w), _p(da), dt, _p(dw), _p(dS), _p(dq), _p(dK),
        _p(dV) if want_dv else None), "pkm_backward")
    return dict(dw=dw, dS=dS, dq=dq, dK=dK, dV=dV)


def full_scores(s_half, ids, n: int):
    """S(id) = s1[id // n] + s2[id % n] for row ids ``ids`` [T,H,m], given
    the half scores ``s_half`` [T,H,2,n] of ``half_scores``."""
    ids = np.asarray(ids, dtype=np.int64)
    a, b = ids // n, ids % n
    return (np.take_along_axis(s_half[:, :, 0], a, -1)
            + np.take_along_axis(s_half[:, :, 1], b, -1))


def value_grad_rows(idx, w, dy, rows):
    """dV[r] = sum over slots with idx == r of w * dy[t], for the row ids
    ``rows`` only; idx/w [T,H,k], dy [T, d_v]."""
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    da, dt = _input(dy)
    T, H, k = idx.shape
    dv = da.shape[1]
    out = np.empty((rows.shape[0], dv))
    _check(_load().orc_value_grad_rows(T, H, k, dv, _p(idx), _p(w), _p(da), dt, _p(rows),
                                       rows.shape[0], _p(out)), "value_grad_rows")
    return out


def sparse_sgd(table, rows, grads, lr):
    """table[r] -= lr * grad for the touched rows only ("모델 안의 메모리":
    a fact lives in a few slots, so only those slots are updated).  fp64,
    returns the updated table (a copy)."""
    t = np.array(table, dtype=np.float64, copy=True)
    rows = np.asarray(rows, dtype=np.int64)
    g = np.asarray(grads, dtype=np.float64)
    for i, r in enumerate(rows):
        t[r] -= lr * g[i]
    return t


def sparse_adam(table, m, v, rows, grads, lr, beta1, beta2, eps, step):
    """Adam restricted to the touched rows (moments of untouched rows are
    left as they are, not decayed), with the bias corrections of the global
    1-based step.  fp64; returns (table, m, v) updated copies."""
    t = np.array(table, dtype=np.float64, copy=True)
    m = np.array(m, dtype=np.float64, copy=True)
    v = np.array(v, dtype=np.float64, copy=True)
    rows = np.asarray(rows, dtype=np.int64)
    g = np.asarray(grads, dtype=np.float64)
    c1 = 1.0 - beta1 ** step
    c2 = 1.0 - beta2 ** step
    for i, r in enumerate(rows):
        m[r] = beta1 * m[r] + (1.0 - beta1) * g[i]
        v[r] = beta2 * v[r] + (1.0 - beta2) * g[i] * g[i]
        t[r] -= lr * (m[r] / c1) / (np.sqrt(v[r] / c2) + eps)
    return t, m, v


ENGRAM_PAD = 0xFFFFFFFF
ENGRAM_EPS = 1e-6


def engram_rows(tokens, orders, K: int, seeds, M):
    """Engram multi-head hashing ("Conditional Memory via Scalable Lookup"
    review, "다중 헤드 해싱"; "핵심 수식" 1: e = E_{n,k}[phi_{n,k}(g_{t,n})]).

    tokens [n_seq, L] ids >= 0; orders: the n-gram orders; K hashes per
    order; seeds / M: per head j = o*K + k (uint64 seed, rows of its
    table).  Returns rows int64 [n_seq*L, len(orders)*K] of the stacked
    table (head j's rows follow those of the heads before it).  The hash is
    the one the C source defines (the page names none)."""
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    n_seq, L = tok.shape
    od = np.ascontiguousarray(orders, dtype=np.int32)
    sd = np.ascontiguousarray(seeds, dtype=np.uint64)
    Ma = np.ascontiguousarray(M, dtype=np.int64)
    HK = len(od) * K
    assert sd.shape == (HK,) and Ma.shape == (HK,)
    rows = np.empty((n_seq * L, HK), dtype=np.int64)
    _check(_load().orc_engram_rows(n_seq, L, _p(tok), len(od), _p(od), K, _p(sd), _p(Ma),
                                   _p(rows)), "engram_rows")
    return rows


def engram_gate(rows, E, h, eps: float = ENGRAM_EPS):
    """e_t = sum of the heads' rows; the context gate ("핵심 수식" 2)
    alpha_t = sigmoid(<RMSNorm(h_t), RMSNorm(e_t)> / sqrt(d)) with the
    parameter-free RMSNorm; v_t = alpha_t e_t.  fp64.  Returns dict(e,
    alpha, v)."""
    r = np.ascontiguousarray(rows, dtype=np.int64)
    T, HK = r.shape
    ea, et = _input(E)
    ha, ht = _input(h)
    d = ea.shape[1]
    e = np.empty((T, d))
    a = np.empty(T)
    v = np.empty((T, d))
    _check(_load().orc_engram_gate(T, HK, d, _p(r), _p(ea), et, ea.shape[0], _p(ha), ht, eps,
                                   _p(e), _p(a), _p(v)), "engram_gate")
    return dict(e=e, alpha=a, v=v)
