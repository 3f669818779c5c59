"""Parity rules between the CUDA path and the CPU oracle (test helpers).

Selection (per token and head): the GPU's index list G must equal the
oracle's O, except where scores tie within rounding.  With s(.) the oracle's
fp64 full score of any row id and tol(x, y) = 1e-5 * max(|x|, |y|, 1):
  * sorted score vectors of G and O agree elementwise within tol, and
  * every id of G not in O scores at least s_k(O) - tol.
This is "bit-exact unless the oracle's k-th and (k+1)-th scores differ by
less than 1e-5 relative", extended to ties at a per-half boundary.

Outputs: |gpu - ref| <= rtol * |ref| + rtol * RMS(ref) elementwise, with
rtol 2e-2 for bf16 and 1e-5 for fp32.  The reference output is the oracle's
fp64 result over the GPU's (validated) index sets, so that a legitimate
tie-swap is compared against the rows actually summed.
"""

from __future__ import annotations

import numpy as np

RTOL = {"bf16": 2e-2, "f32": 1e-5}
# Weights: the GPU scores carry fp32 rounding of a d_half-long dot product
# (|dS| <= ~2e-5 absolute at the sizes used); a softmax weight moves by at
# most ~2|dS| relative.
W_RTOL = {"bf16": 1e-4, "f32": 5e-5}
SEL_TOL = 1e-5


def _tol(x, y):
    return SEL_TOL * np.maximum(np.maximum(np.abs(x), np.abs(y)), 1.0)


def check_selection(idx_gpu, idx_orc, s_half, n):
    """Apply the acceptance rule.  Returns the number of (t, h) exempted.

    idx_gpu, idx_orc [T,H,k] (int); s_half [T,H,2,n] oracle half scores."""
    import oracle

    G = np.asarray(idx_gpu, dtype=np.int64)
    O = np.asarray(idx_orc, dtype=np.int64)
    assert G.shape == O.shape
    T, H, k = G.shape
    N = n * n
    assert G.min() >= 0 and G.max() < N, "row id out of range"
    srt = np.sort(G, axis=-1)
    assert np.all(srt[..., 1:] != srt[..., :-1]), "duplicate row id in a selection"
    sG = oracle.full_scores(s_half, G, n)
    sO = oracle.full_scores(s_half, O, n)
    same = np.all(G == O, axis=-1)
    exempt = 0
    for t, h in zip(*np.nonzero(~same)):
        g, o = sG[t, h], sO[t, h]
        a, b = np.sort(g), np.sort(o)
        assert np.all(np.abs(a - b) <= _tol(a, b)), \
            f"(t={t}, h={h}) score vectors differ: gpu {G[t, h]} oracle {O[t, h]}"
        extra = np.setdiff1d(G[t, h], O[t, h])
        kth = o.min()
        for r in extra:
            sr = oracle.full_scores(s_half[t:t + 1, h:h + 1], np.array([[[r]]]), n)[0, 0, 0]
            assert sr >= kth - _tol(sr, kth), f"(t={t}, h={h}) row {r} below the k-th score"
        # the GPU order must follow its scores (ties within tol allowed)
        assert np.all(np.diff(g) <= _tol(g[1:], g[:-1])), f"(t={t}, h={h}) not sorted"
        exempt += 1
    return exempt


def close(gpu, ref, rtol, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(gpu - ref)
    bound = rtol * np.abs(ref) + rtol * rms
    bad = err > bound
    assert not np.any(bad), (
        f"{what}: {int(bad.sum())} of {bad.size} outside rtol {rtol}; "
        f"max abs err {err.max():.3g}, rms(ref) {rms:.3g}")
    return float(err.max() / max(rms, 1e-30))


def weights_close(w_gpu, w_ref, rtol, what="weights"):
    w_gpu = np.asarray(w_gpu, dtype=np.float64)
    w_ref = np.asarray(w_ref, dtype=np.float64)
    err = np.abs(w_gpu - w_ref)
    bad = err > rtol * np.abs(w_ref) + 1e-7
    assert not np.any(bad), f"{what}: {int(bad.sum())} bad, max rel {np.max(err / np.abs(w_ref)):.3g}"
    np.testing.assert_allclose(w_gpu.sum(-1), 1.0, atol=1e-5)


def forward_reference(q, K, k, idx_gpu, table_rows, row_ids, n, x=None, W1=None, W2=None):
    """Oracle selection + checks + the oracle's output over the GPU's sets.

    ``table_rows`` holds the value rows ``row_ids`` (sorted unique ids that
    cover every GPU-selected row).  Returns dict(idx_orc, w_ref, out_ref,
    exempt)."""
    import oracle

    idx_o, S_o, w_o, _ = oracle.pkm_select(q, K, k)
    s_half = oracle.half_scores(q, K)
    exempt = check_selection(idx_gpu, idx_o, s_half, n)
    G = np.asarray(idx_gpu, dtype=np.int64)
    sG = oracle.full_scores(s_half, G, n)
    w_ref = oracle.softmax(sG)
    pos = np.searchsorted(row_ids, G)
    assert np.all(row_ids[pos] == G)
    T, H, kk = G.shape
    y = oracle.bag(pos.reshape(T, H * kk), w_ref.reshape(T, H * kk), table_rows)
    out = y if x is None else oracle.memplus(y, x, W1, W2)
    return dict(idx_orc=idx_o, w_ref=w_ref, out_ref=out, exempt=exempt, y_ref=y)
