"""GPU parity of the reduced projection with int8 weights (rmm_linear_int8):
the selection on the bf16 activations, then (A[:, I] Wq[I, :]) * scale from the
kept int8 rows only.  References: the oracle's TopK for the index set and
oracle.int8_product_rows on the library's own set for the product."""
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


def int8_parity(A, Wq, s, rho):
    Y, idx = rmm.linear_int8(A.cuda(), Wq.cuda(), s.cuda(), rho, return_idx=True)
    torch.cuda.synchronize()
    Aw = synthetic.widen(A)
    I = idx.cpu().numpy().astype(np.int64)
    check_index_set(I, oracle.column_sq_norms(Aw), oracle.retention_count(rho, A.shape[1]),
                    f"int8 n={A.shape[0]} d={A.shape[1]} rho={rho}")
    ref = oracle.int8_product_rows(Aw, Wq.numpy(), s.numpy(), I)
    check_close(synthetic.widen(Y.cpu()), ref, "int8 product")
    return Y, idx


@pytest.mark.parametrize("n", [1, 2, 3, 8, 16, 17, 32])
@pytest.mark.parametrize("rho", [0.5, 0.7, 1.0])
def test_int8_small_ragged(n, rho):
    """d and m off the 2048-column block, the 512-column super tile and the 16-row
    unroll (d = 1000, m = 2056: the last 16-byte int8 chunk holds 8 columns); n = 1, 2
    on the CUDA cores, n >= 3 on the tensor cores."""
    g = synthetic.rng(37)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, 1000, 1.5))
    Wq, s = synthetic.int8_weight(g, 1000, 2056)
    int8_parity(A, Wq, s, rho)


def test_int8_matches_the_oracle_entry_point_and_repeats():
    g = synthetic.rng(38)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 4, 512, 1.5))
    Wq, s = synthetic.int8_weight(g, 512, 1024)
    Y1, I1 = rmm.linear_int8(A.cuda(), Wq.cuda(), s.cuda(), 0.5, return_idx=True)
    Y2 = rmm.linear_int8(A.cuda(), Wq.cuda(), s.cuda(), 0.5)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    ref = oracle.rmm_linear_int8(synthetic.widen(A), Wq.numpy(), s.numpy(), 0.5)
    assert np.array_equal(I1.cpu().numpy(), ref["I"])
    check_close(synthetic.widen(Y1.cpu()), ref["Y"], "int8 entry point")


def test_int8_extreme_codes_and_scales_are_exact():
    """Codes -127, 0 and 127 and powers-of-two scales: with one kept row of a one-row
    activation of value 1, Y must be the code times the scale exactly."""
    A = torch.zeros((1, 64), dtype=torch.bfloat16)
    A[0, 5] = 1.0
    Wq = torch.zeros((64, 16), dtype=torch.int8)
    Wq[5] = torch.tensor([-127, 127, 0, 1, -1, 64, -64, 100, -100, 3, -3, 5, -5, 7, -7, 126], dtype=torch.int8)
    s = torch.tensor([2.0 ** (-e) for e in range(16)], dtype=torch.float32)
    Y, idx = rmm.linear_int8(A.cuda(), Wq.cuda(), s.cuda(), 1 / 64, return_idx=True)
    torch.cuda.synchronize()
    assert idx.cpu().tolist() == [5]
    expect = (Wq[5].double() * s.double()).to(torch.bfloat16)
    assert torch.equal(Y.cpu()[0], expect)


@pytest.mark.parametrize("n", [1, 8, 32])
def test_int8_70b_mlp_up(n):
    """Llama-3.1-70B MLP-up shape (d = 8192, m = 28672) with int8 weights."""
    g = synthetic.rng(39)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, 8192, 1.5))
    Wq, s = synthetic.int8_weight(g, 8192, 28672)
    int8_parity(A, Wq, s, 0.5)


def test_int8_tensor_cores_match_the_cuda_core_kernel_row_by_row():
    """The same weights and rows through both kernels: the tensor-core product of 8
    rows equals, row by row, the CUDA-core product of each row alone within the
    parity tolerance (both accumulate in fp32 from exact int8 values)."""
    g = synthetic.rng(47)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 8, 2048, 1.5))
    Wq, s = synthetic.int8_weight(g, 2048, 4096)
    Ad, Wd, sd = A.cuda(), Wq.cuda(), s.cuda()
    Y8 = rmm.linear_int8(Ad, Wd, sd, 1.0)
    torch.cuda.synchronize()
    for r in range(8):
        Y1 = rmm.linear_int8(Ad[r:r + 1].contiguous(), Wd, sd, 1.0)
        torch.cuda.synchronize()
        check_close(synthetic.widen(Y8[r:r + 1].cpu()), synthetic.widen(Y1.cpu()), f"row {r}")
