"""The decode selection in one cluster launch (scores, TopK, index set and
x[:, I] for n <= 32 rows, d <= 16384) against the three-kernel selection
(rmm_select) and the oracle.

Both selections rank bit-identical fp64 scores with an exact radix select, so
their index sets must be equal, element for element, on every shape, rho and
tie pattern; the reduced product that consumes the packed x[:, I] is checked
against the oracle on the library's own set."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check_close, check_index_set

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")


@pytest.fixture(scope="module", autouse=True)
def built():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    yield
    assert rmm.device_error() == 0


def fused_vs_select(A, m=64, rho=0.5, seed=0):
    """rmm_linear's decode path (fused selection) vs rmm_select on the same x."""
    n, d = A.shape
    g = synthetic.rng(seed + 7)
    B = synthetic.to_bf16(synthetic.gaussian_weight(g, d, m))
    ld = (d + 7) // 8 * 8
    Ad = torch.zeros((n, ld), dtype=torch.bfloat16, device="cuda")
    Ad[:, :d].copy_(A)
    Ad = Ad[:, :d]
    Bd = B.cuda()
    Y, idx = rmm.linear(Ad, Bd, rho, return_idx=True)
    ref, cs, _ = rmm.select(Ad, rho)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref), "fused decode selection differs from rmm_select"
    I = idx.cpu().numpy().astype(np.int64)
    Aw = synthetic.widen(A)
    check_index_set(I, oracle.column_sq_norms(Aw), oracle.retention_count(rho, d), f"decode select n={n} d={d} rho={rho}")
    check_close(synthetic.widen(Y.cpu()), oracle.rmm_linear_rows(Aw, synthetic.widen(B), I, np.arange(n)),
                f"decode product n={n} d={d} rho={rho}")
    return idx


SHAPES = [(1, 12), (1, 1000), (3, 2048), (8, 2049), (8, 8192), (17, 4100), (32, 8192), (1, 16384), (32, 14336),
          (5, 16384), (2, 16383)]


@pytest.mark.parametrize("n,d", SHAPES)
@pytest.mark.parametrize("rho", [0.05, 0.5, 0.9, 1.0])
def test_fused_decode_selection_matches_select(n, d, rho):
    g = synthetic.rng(3000 + n * 17 + d)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, d, 1.5))
    fused_vs_select(A, rho=rho, seed=n + d)


@pytest.mark.parametrize("d", [1000, 8192, 16384])
def test_fused_decode_selection_exact_ties(d):
    """One row of values from a small set (most squares tie exactly), all-equal
    rows, and duplicated columns with zero columns: the lower-index rule decides."""
    g = synthetic.rng(d + 5)
    vals = np.array([0.5, 1.0, 1.5, 2.0, -0.5, -1.0, -2.0, 0.0], np.float32)
    A = synthetic.to_bf16(vals[g.integers(0, vals.size, size=(1, d))])
    for rho in (0.1, 0.3, 0.5, 0.77, 0.95):
        fused_vs_select(A, rho=rho, seed=d)
    ones = torch.ones((4, d), dtype=torch.bfloat16)
    for rho in (0.1, 0.5):
        idx = fused_vs_select(ones, rho=rho, seed=d)
        assert idx.cpu().tolist() == list(range(oracle.retention_count(rho, d)))
    half = synthetic.outlier_activations(g, 6, d // 4, 1.0)
    A = synthetic.to_bf16(np.concatenate([half, half, np.zeros((6, d - 2 * (d // 4)), np.float32)], axis=1))
    for rho in (0.3, 0.5, 0.6):
        fused_vs_select(A, rho=rho, seed=d + 1)


@pytest.mark.parametrize("n", [8, 32])
def test_fused_decode_selection_low_word_keys(n):
    """Scores 1 + s_j with s_j < 2^-30: every key shares its high word and the
    order lives in the low word (repeats of s_j tie exactly)."""
    d = 8192
    g = synthetic.rng(n * 11 + 3)
    A = np.zeros((n, d), np.float32)
    A[0, :] = 1.0
    A[n // 2, :] = np.float32(2.0 ** -20) * (1.0 + g.integers(0, 128, size=d) / 128.0)
    A = synthetic.to_bf16(A)
    for rho in (0.25, 0.5, 0.9):
        fused_vs_select(A, rho=rho, seed=n)


def test_wide_decode_rows_use_the_three_kernel_chain():
    """d = 20000 is beyond the fused kernel's 16384 columns: the chain of score,
    selection and pack kernels runs, with the same result contract."""
    g = synthetic.rng(99)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 4, 20000, 1.5))
    fused_vs_select(A, rho=0.5, seed=1)
