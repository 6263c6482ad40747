"""Shared parity checks: CUDA path vs the CPU oracle.

Acceptance (the tolerances stated for bf16 inputs with fp32 accumulation):
  * index sets: size k, strictly ascending, in range, and equal to the oracle's
    except for indices inside the near-tie band (norms within 1e-5 relative of
    the k-th largest), where either choice is correct; such differences are
    counted and returned so the caller can log them;
  * products: relative Frobenius error <= 1e-2 and max-abs error <=
    3e-2 * max|Y_ref|, with Y_ref the oracle's float64 product on the GPU's own
    index set; -inf positions (masked scores) must match exactly.
"""
import numpy as np

import oracle

REL_FRO = 1e-2
MAX_ABS_FRAC = 3e-2
TIE_BAND = 1e-5


# Every index-set comparison is recorded here as (what, k, near-tie differences);
# tests/conftest.py prints the totals at the end of the session.
NEAR_TIE_LOG = []
MAX_TIES = 2


def check_index_set(I_gpu, q_ref, k, what="", max_ties=MAX_TIES):
    """Compare the library's index set with the oracle's TopK of the oracle's scores.

    Differences are allowed only inside the near-tie band; their number (each swap
    counts once) is logged, printed when non-zero, bounded by ``max_ties`` and
    returned."""
    I = np.asarray(I_gpu, dtype=np.int64).reshape(-1)
    q_ref = np.asarray(q_ref, dtype=np.float64)
    d = q_ref.shape[0]
    assert I.shape == (k,), (I.shape, k)
    assert np.all(np.diff(I) > 0), "index set is not strictly ascending"
    assert I[0] >= 0 and I[-1] < d, "index out of range"
    s = np.sqrt(q_ref)
    ref = oracle.topk_ascending(s, k)
    diff = set(I.tolist()) ^ set(ref.tolist())
    if diff:
        band = set(oracle.near_tie_band(s, k, TIE_BAND).tolist())
        outside = sorted(diff - band)
        assert not outside, f"index sets differ outside the near-tie band at {outside[:10]}"
    ties = len(diff) // 2
    NEAR_TIE_LOG.append((what, k, ties))
    if ties:
        print(f"near-tie differences: {ties} of k={k} ({what})")
    assert ties <= max_ties, f"{what}: {ties} near-tie differences (bound {max_ties})"
    return ties


def check_close(Y_gpu, Y_ref, what=""):
    Y = np.asarray(Y_gpu, dtype=np.float64)
    R = np.asarray(Y_ref, dtype=np.float64)
    assert Y.shape == R.shape, (Y.shape, R.shape)
    ninf_r = np.isneginf(R)
    assert np.array_equal(np.isneginf(Y), ninf_r), f"{what}: -inf mask differs"
    fin = ~ninf_r
    assert np.all(np.isfinite(Y[fin])), f"{what}: non-finite values"
    Yf, Rf = Y[fin], R[fin]
    if Rf.size == 0:
        return 0.0, 0.0
    nref = float(np.linalg.norm(Rf))
    err = float(np.linalg.norm(Yf - Rf))
    mx = float(np.max(np.abs(Rf)))
    mabs = float(np.max(np.abs(Yf - Rf)))
    if nref == 0.0:
        assert err == 0.0, f"{what}: expected exact zeros"
        return 0.0, 0.0
    assert err <= REL_FRO * nref, f"{what}: relative Frobenius error {err / nref:.3e}"
    assert mabs <= MAX_ABS_FRAC * mx, f"{what}: max-abs error {mabs:.3e} vs max {mx:.3e}"
    return err / nref, mabs / mx


def check_colsq(q_gpu, q_ref, rel=2e-6):
    q = np.asarray(q_gpu, dtype=np.float64)
    r = np.asarray(q_ref, dtype=np.float64)
    scale = np.maximum(np.abs(r), 1e-300)
    bad = np.abs(q - r) > rel * scale
    assert not np.any(bad & (r > 0)), f"column sums of squares off at {np.nonzero(bad)[0][:10]}"
    assert np.all(q[r == 0] == 0)


def device_padded(t, mult=8):
    """Copy a 2-D CPU tensor to the GPU in a buffer whose row stride is a multiple of
    ``mult`` elements (the library's leading-dimension rule); returns the view."""
    import torch
    rows, cols = t.shape
    ld = (cols + mult - 1) // mult * mult
    buf = torch.zeros((rows, ld), dtype=t.dtype, device="cuda")
    buf[:, :cols].copy_(t)
    return buf[:, :cols]
