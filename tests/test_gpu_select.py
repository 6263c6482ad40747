"""GPU parity of the column scores and TopK selection (rmm_select) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check_colsq, check_index_set, device_padded

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")


@pytest.fixture(scope="module", autouse=True)
def built():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    yield
    assert rmm.device_error() == 0


def run_select(A_cpu, rho, causal=False):
    A = device_padded(A_cpu)
    idx, cs, rt = rmm.select(A, rho, causal=causal)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cs.cpu().numpy(), rt.cpu().numpy()


SHAPES = [(1, 12), (7, 100), (16, 1024), (128, 1024), (33, 4095), (300, 2000), (5, 16384), (64, 32768)]


@pytest.mark.parametrize("n,d", SHAPES)
@pytest.mark.parametrize("rho", [0.5, 0.7, 0.9, 1.0])
def test_select_random_shapes(n, d, rho):
    g = synthetic.rng(1000 + n * 7 + d)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, d, 1.5))
    idx, cs, rt = run_select(A, rho)
    Aw = synthetic.widen(A)
    q = oracle.column_sq_norms(Aw)
    check_colsq(cs, q)
    k = oracle.retention_count(rho, d)
    ties = check_index_set(idx, q, k)
    assert ties <= 2
    I_ref = oracle.topk_ascending(np.sqrt(q), k)
    assert abs(rt - oracle.retained_energy(q, I_ref)) < 1e-6


def test_select_ties_pick_lowest_indices():
    for d in (12, 1000, 4096, 16384):
        A = torch.ones((3, d), dtype=torch.bfloat16)
        for rho in (0.1, 0.5, 0.9):
            idx, _, _ = run_select(A, rho)
            k = oracle.retention_count(rho, d)
            assert idx.tolist() == list(range(k))


def test_select_duplicate_columns_and_zeros():
    g = synthetic.rng(77)
    base = synthetic.outlier_activations(g, 9, 40, 1.0)
    A = np.concatenate([base, base, np.zeros((9, 40), np.float32)], axis=1)  # exact duplicates + zero columns
    A = synthetic.to_bf16(A)
    for rho in (0.3, 0.5, 0.6, 0.8, 0.95):
        idx, cs, _ = run_select(A, rho)
        q = oracle.column_sq_norms(synthetic.widen(A))
        k = oracle.retention_count(rho, 120)
        # duplicated columns have bitwise-equal scores on both sides: exact match required
        assert idx.tolist() == oracle.topk_ascending(np.sqrt(q), k).tolist()


def test_select_k1_is_argmax():
    g = synthetic.rng(5)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 20, 3000, 1.5))
    idx, _, _ = run_select(A, 1e-6)
    q = oracle.column_sq_norms(synthetic.widen(A))
    assert idx.tolist() == [int(np.argmax(q))]


def test_select_causal_masks_upper_triangle():
    g = synthetic.rng(9)
    n, d = 300, 520
    logits = 2.0 * g.standard_normal((n, d), dtype=np.float32)
    P = synthetic.causal_softmax_rows(logits, offset=d - n)
    junk = np.triu(np.full((n, d), 7.0, np.float32), d - n + 1)  # garbage above the diagonal
    Pt = synthetic.to_bf16(P + junk)
    for rho in (0.5, 0.8):
        idx, cs, _ = run_select(Pt, rho, causal=True)
        q = oracle.column_sq_norms(synthetic.widen(Pt), causal=True)
        check_colsq(cs, q)
        check_index_set(idx, q, oracle.retention_count(rho, d))


def test_select_batched_heads():
    Q, _ = synthetic.qk_inputs(hq=8, hkv=2, n=512)
    A = Q[0].cuda()
    idx, cs, _ = rmm.select(A, 0.7)
    torch.cuda.synchronize()
    Qw = synthetic.widen(Q)[0]
    for h in range(8):
        q = oracle.column_sq_norms(Qw[h])
        check_colsq(cs[h].cpu().numpy(), q)
        check_index_set(idx[h].cpu().numpy(), q, 90)


def test_select_deterministic():
    g = synthetic.rng(3)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 4096, 4096, 1.5)).cuda()
    a = rmm.select(A, 0.7)
    b = rmm.select(A, 0.7)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------------- the radix passes themselves
# Given the GPU's own scores, the TopK rule has one answer: the index set must be
# exactly oracle.topk_ascending of those scores (no near-tie allowance).  Shapes
# cover both column-score kernels (at most 32 rows, and 64 rows or more) and every
# launch shape of the selection kernel.
OWN_SHAPES = [(1, 12), (3, 200), (8, 1000), (16, 2048), (32, 4096), (1, 8192), (8, 8192), (32, 8192),
              (5, 16384), (64, 256), (64, 1024), (96, 4096), (64, 8192), (70, 14336), (64, 32768)]


@pytest.mark.parametrize("n,d", OWN_SHAPES)
@pytest.mark.parametrize("rho", [0.05, 0.5, 0.9])
def test_select_exact_on_own_scores(n, d, rho):
    g = synthetic.rng(2000 + n * 13 + d)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, d, 1.5))
    idx, cs, rt = run_select(A, rho)
    k = oracle.retention_count(rho, d)
    assert idx.tolist() == oracle.topk_ascending(cs, k).tolist()
    assert abs(rt - oracle.retained_energy(cs, idx)) < 1e-12


@pytest.mark.parametrize("d", [1000, 4096, 8192, 16384])
def test_select_single_row_exact_ties(d):
    """One row of values from a small set: most scores tie exactly (the squares of
    equal magnitudes), so the lower-index rule decides most of the set."""
    g = synthetic.rng(d + 11)
    vals = np.array([0.5, 1.0, 1.5, 2.0, -0.5, -1.0, -2.0, 0.0], np.float32)
    A = synthetic.to_bf16(vals[g.integers(0, vals.size, size=(1, d))])
    q = oracle.column_sq_norms(synthetic.widen(A))
    for rho in (0.1, 0.3, 0.5, 0.77, 0.95):
        idx, cs, _ = run_select(A, rho)
        k = oracle.retention_count(rho, d)
        np.testing.assert_array_equal(cs, q)  # exact squares
        assert idx.tolist() == oracle.topk_ascending(q, k).tolist()


@pytest.mark.parametrize("n,row_small", [(8, 4), (32, 20), (64, 40)])
def test_select_keys_differing_only_in_low_word(n, row_small):
    """Every score is 1 + s_j with s_j < 2^-30: the top 32 bits of all fp64 keys are
    equal and the order lives in the low word (and repeats of s_j tie exactly)."""
    d = 2048
    g = synthetic.rng(n * 5 + 1)
    A = np.zeros((n, d), np.float32)
    A[0, :] = 1.0
    m = g.integers(0, 128, size=d)
    A[row_small, :] = np.float32(2.0 ** -20) * (1.0 + m / 128.0)
    A = synthetic.to_bf16(A)
    q = oracle.column_sq_norms(synthetic.widen(A))
    assert np.all((q.view(np.uint64) >> 32) == (q[0].view(np.uint64) >> 32))
    for rho in (0.25, 0.5, 0.9):
        idx, cs, _ = run_select(A, rho)
        k = oracle.retention_count(rho, d)
        assert idx.tolist() == oracle.topk_ascending(cs, k).tolist()
        if n <= 32:
            # fp32 groups of four rows keep 1 and s_j apart, so the keys are exact
            np.testing.assert_array_equal(cs, q)
            assert idx.tolist() == oracle.topk_ascending(q, k).tolist()


def test_select_short_batched_strided():
    """Batched short matrices with a padded row stride and batch stride (the
    decode query-group layout): every item's scores and index set are its own."""
    g = synthetic.rng(404)
    batch, n, d, lda = 5, 4, 1000, 1016
    base = synthetic.to_bf16(synthetic.outlier_activations(g, batch * n, lda, 1.0)).reshape(batch, n, lda)
    A = base.cuda()[:, :, :d]
    idx, cs, _ = rmm.select(A, 0.4)
    torch.cuda.synchronize()
    for b in range(batch):
        q = oracle.column_sq_norms(synthetic.widen(base[b, :, :d]))
        check_colsq(cs[b].cpu().numpy(), q)
        k = oracle.retention_count(0.4, d)
        assert idx[b].cpu().tolist() == oracle.topk_ascending(cs[b].cpu().numpy(), k).tolist()
