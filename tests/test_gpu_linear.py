"""GPU parity of rmm_linear (column norms -> TopK -> pack -> tcgen05 gathered GEMM)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check_close, check_index_set, device_padded

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")


@pytest.fixture(scope="module", autouse=True)
def built():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    yield
    assert rmm.device_error() == 0


def parity_linear(A, B, rho, rows=None):
    """Run the CUDA path and compare with the oracle (all rows, or sampled ``rows``)."""
    Ad, Bd = device_padded(A), device_padded(B)
    Y = device_padded(torch.zeros((A.shape[0], B.shape[1]), dtype=torch.bfloat16))
    Y, idx = rmm.linear(Ad, Bd, rho, out=Y, return_idx=True)
    torch.cuda.synchronize()
    Aw, Bw = synthetic.widen(A), synthetic.widen(B)
    q = oracle.column_sq_norms(Aw)
    k = oracle.retention_count(rho, A.shape[1])
    I = idx.cpu().numpy().astype(np.int64)
    ties = check_index_set(I, q, k, f"linear n={A.shape[0]} d={A.shape[1]} m={B.shape[1]} rho={rho}")
    if rows is None:
        ref = oracle.reduced_product(Aw, Bw, I)
        got = synthetic.widen(Y.cpu())
    else:
        ref = oracle.rmm_linear_rows(Aw, Bw, I, rows)
        got = synthetic.widen(Y[torch.as_tensor(rows, device=Y.device)].cpu())
    check_close(got, ref, f"linear n={A.shape[0]} d={A.shape[1]} m={B.shape[1]} rho={rho}")
    return Y, idx, ties


def test_linear_single_layer_128x1024():
    A, B = synthetic.linear_small()
    Y, idx, _ = parity_linear(A, B, 0.5)
    assert idx.numel() == 512
    # independent second reference: cuBLAS on the GPU's own index set
    I = idx.long()
    Ad, Bd = A.cuda(), B.cuda()
    ref = (Ad[:, I].float() @ Bd[I, :].float())
    err = (Y.float() - ref).norm() / ref.norm()
    assert err.item() < 1e-2
    # bitwise determinism
    Y2, idx2 = rmm.linear(Ad, Bd, 0.5, return_idx=True)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(Y, Y2)


SMALL = [(1, 12, 8), (5, 64, 64), (130, 200, 72), (257, 1000, 300), (128, 1024, 1024), (300, 2056, 520),
         (64, 4096, 4096 + 8)]


@pytest.mark.parametrize("n,d,m", SMALL)
@pytest.mark.parametrize("rho", [0.5, 0.7, 1.0])
def test_linear_ragged_shapes(n, d, m, rho):
    g = synthetic.rng(n * 131 + d * 7 + m)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, d, 1.5))
    B = synthetic.to_bf16(synthetic.gaussian_weight(g, d, m))
    parity_linear(A, B, rho)


def test_linear_k1_and_tiny_rho():
    g = synthetic.rng(21)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 40, 333, 1.5))
    B = synthetic.to_bf16(synthetic.gaussian_weight(g, 333, 96))
    Y, idx, _ = parity_linear(A, B, 1e-4)
    assert idx.numel() == 1


def test_linear_strided_operands():
    g = synthetic.rng(23)
    Abig = synthetic.to_bf16(synthetic.outlier_activations(g, 200, 1040, 1.5)).cuda()
    Bbig = synthetic.to_bf16(synthetic.gaussian_weight(g, 1000, 264)).cuda()
    A = Abig[:, :1000]          # lda = 1040
    B = Bbig[:, :256]           # ldb = 264
    Ybig = torch.zeros((200, 272), dtype=torch.bfloat16, device="cuda")
    Y = Ybig[:, :256]           # ldy = 272
    rmm.linear(A, B, 0.6, out=Y)
    torch.cuda.synchronize()
    Aw, Bw = synthetic.widen(A.cpu()), synthetic.widen(B.cpu())
    I, _, _ = oracle.select(Aw, 0.6)
    check_close(synthetic.widen(Y.cpu()), oracle.reduced_product(Aw, Bw, I), "strided")
    assert torch.count_nonzero(Ybig[:, 256:]).item() == 0


def test_linear_identity_weight_keeps_selected_columns():
    g = synthetic.rng(29)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, 64, 256, 1.0))
    B = torch.eye(256, dtype=torch.bfloat16)
    Y, idx = rmm.linear(A.cuda(), B.cuda(), 0.5, return_idx=True)
    torch.cuda.synchronize()
    expect = torch.zeros_like(A)
    I = idx.cpu().long()
    expect[:, I] = A[:, I]
    assert torch.equal(Y.cpu(), expect)


_PREFILL = {}


def prefill_inputs(name):
    """One projection's seeded inputs, drawn once for all rho values of the test."""
    if name not in _PREFILL:
        _PREFILL.clear()
        _PREFILL[name] = synthetic.prefill_projection(name)
    return _PREFILL[name]


@pytest.mark.parametrize("rho", [0.5, 0.7, 0.9, 1.0])
@pytest.mark.parametrize("name", ["q_proj", "gate_proj", "up_proj", "down_proj"])
def test_linear_llama8b_prefill_sampled(name, rho):
    """Full-size Llama-3.1-8B projection shapes (n = 4096) at every rho of the
    workload, sampled output rows against oracle.rmm_linear_rows on the library's
    index set (which is checked against the oracle's first)."""
    A, W = prefill_inputs(name)
    rows = np.concatenate([np.arange(0, 4096, 97), [4095]])
    parity_linear(A, W, rho, rows=rows)


@pytest.mark.parametrize("n", [300, 100])
def test_stage_entry_points_compose_to_rmm_linear(n):
    """rmm_select -> rmm_gather_columns -> rmm_gemm_gathered (n > 128), or
    -> rmm_gather_rows -> rmm_gemm_packed (n <= 128), gives the same bits as
    rmm_linear; and the gathered product equals the packed one bit for bit (the
    same k-blocks in the same order, only the source of B's rows differs)."""
    g = synthetic.rng(31)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, 1000, 1.5)).cuda()
    B = synthetic.to_bf16(synthetic.gaussian_weight(g, 1000, 520)).cuda()
    Y, idx = rmm.linear(A, B, 0.7, return_idx=True)
    idx2, _, _ = rmm.select(A, 0.7)
    k = idx2.numel()
    ap = rmm.gather_columns(A, idx2, ld_pack=712)
    bp = rmm.gather_rows(B, idx2, ld_pack=528)
    Y2 = rmm.gemm_packed(ap, k, bp, 520)
    Y3 = rmm.gemm_gathered(ap, k, B, idx2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(Y, Y3 if n > 128 else Y2)
    if n > 128:
        assert torch.equal(Y2, Y3)
    I = idx2.cpu().long()
    expect = torch.zeros((n, 712), dtype=torch.bfloat16)
    expect[:, :k] = A.cpu()[:, I]
    assert torch.equal(ap.cpu(), expect)
    assert torch.equal(bp.cpu()[:, :520], B.cpu()[I, :])


def _bf16_rows(g, rows, cols):
    return synthetic.to_bf16(g.standard_normal((rows, cols), dtype=np.float32))


def test_gather_rows_long_rows_unsorted_indices():
    """Rows of 8200 columns (two bulk chunks, the second 16 bytes), indices in any
    order with repeats; the packed rows are exact copies."""
    g = synthetic.rng(32)
    B = _bf16_rows(g, 3000, 8200).cuda()
    idx = torch.as_tensor(g.integers(0, 3000, size=1700), dtype=torch.int32).cuda()
    bp = rmm.gather_rows(B, idx)
    torch.cuda.synchronize()
    assert torch.equal(bp[:, :8200], B[idx.long()])


def test_gather_rows_more_rows_than_one_wave_holds():
    """650000 kept rows of 16 bytes: more than two CTAs per SM x 2048 rows, so the
    grid grows past two CTAs per SM."""
    g = synthetic.rng(33)
    B = _bf16_rows(g, 700000, 8).cuda()
    idx = torch.as_tensor(np.sort(g.choice(700000, size=650000, replace=False)), dtype=torch.int32).cuda()
    bp = rmm.gather_rows(B, idx)
    torch.cuda.synchronize()
    assert torch.equal(bp, B[idx.long()])


def test_gather_columns_long_strided_rows():
    """Rows of 14336 columns inside a wider allocation (lda 14400), 7000 kept
    columns padded to 7040."""
    g = synthetic.rng(34)
    full = _bf16_rows(g, 37, 14400).cuda()
    A = full[:, :14336]
    idx = torch.as_tensor(np.sort(g.choice(14336, size=7000, replace=False)), dtype=torch.int32).cuda()
    ap = rmm.gather_columns(A, idx, ld_pack=7040)
    torch.cuda.synchronize()
    assert torch.equal(ap[:, :7000], A[:, idx.long()])
    assert not ap[:, 7000:].any()


@pytest.mark.parametrize("n,k,m", [(4096, 1024, 4736), (4000, 1000, 4696), (19072, 576, 256), (256, 200, 512),
                                   (4096, 2048, 14336)])
def test_gemm_packed_narrow_last_wave(n, k, m):
    """Products whose last wave of 128 x 256 output tiles is partial (or that have
    fewer tiles than SMs): those tiles are computed as 2 or 4 narrower pieces along
    N.  Every shape here has such a tail on a 148-SM B200; the product must match
    the fp32 reference within the parity tolerance and repeat bit for bit."""
    g = synthetic.rng(35)
    ldp = (k + 7) // 8 * 8
    A = torch.zeros((n, ldp), dtype=torch.bfloat16)
    A[:, :k] = synthetic.to_bf16(g.standard_normal((n, k), dtype=np.float32))
    B = synthetic.to_bf16(g.standard_normal((k, m), dtype=np.float32) / np.float32(np.sqrt(k)))
    A, B = A.cuda(), B.cuda()
    Y1 = rmm.gemm_packed(A, k, B, m)
    Y2 = rmm.gemm_packed(A, k, B, m)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    ref = (A[:, :k].float() @ B.float()).cpu().numpy()
    check_close(Y1.float().cpu().numpy(), ref, "narrow-last-wave product")
    # every column block of the tail tiles, element by element against the reference
    tail = Y1[-128:, -512:].float().cpu().numpy()
    assert np.abs(tail - ref[-128:, -512:]).max() <= 3e-2 * np.abs(ref).max()


@pytest.mark.parametrize("d,k,ld", [(296, 150, 152), (504, 250, 256), (16, 5, 8)])
def test_gather_columns_short_rows(d, k, ld):
    """Rows of at most 512 columns take the warp-per-row gather without staging;
    k_pad up to 256, kept columns in any order."""
    g = synthetic.rng(44)
    A = synthetic.to_bf16(g.standard_normal((1001, d), dtype=np.float32)).cuda()
    idx = torch.as_tensor(g.permutation(d)[:k], dtype=torch.int32).cuda()
    ap = rmm.gather_columns(A, idx, ld_pack=ld)
    torch.cuda.synchronize()
    assert torch.equal(ap[:, :k], A[:, idx.long()])
    assert not ap[:, k:].any()


@pytest.mark.parametrize("d,k,ld,lda", [(128, 64, 64, 128), (128, 39, 64, 136), (64, 17, 24, 64), (256, 200, 256, 264)])
def test_gather_columns_narrow_rows(d, k, ld, lda):
    """Many rows of 64, 128 or 256 columns (the attention's packed score operands):
    the 8-rows-per-warp staged gather; strided rows, kept columns in any order,
    zero padding past k."""
    g = synthetic.rng(45)
    full = synthetic.to_bf16(g.standard_normal((16384, lda), dtype=np.float32)).cuda()
    A = full[:, :d]
    idx = torch.as_tensor(g.permutation(d)[:k], dtype=torch.int32).cuda()
    ap = rmm.gather_columns(A, idx, ld_pack=ld)
    torch.cuda.synchronize()
    assert torch.equal(ap[:, :k], A[:, idx.long()])
    assert not ap[:, k:].any()


_DECODE_W = {}


def decode_weight():
    if "W" not in _DECODE_W:
        _, _DECODE_W["W"] = synthetic.decode_gemv(1)
    return _DECODE_W["W"]


@pytest.mark.parametrize("n", [1, 8, 32])
@pytest.mark.parametrize("rho", [0.5, 0.7, 0.9, 1.0])
def test_linear_decode_llama70b_mlp_up(n, rho):
    """Decode GEMV on the Llama-3.1-70B MLP-up shape: x n x 8192, W 8192 x 28672."""
    A, _ = synthetic.decode_gemv(n, weight=False)
    parity_linear(A, decode_weight(), rho)


@pytest.mark.parametrize("n,d,m", [(2, 300, 1000), (16, 64, 136), (17, 4100, 264), (31, 1000, 8), (32, 12, 4096)])
@pytest.mark.parametrize("rho", [0.3, 1.0])
def test_linear_decode_ragged(n, d, m, rho):
    g = synthetic.rng(n * 7919 + d * 31 + m)
    A = synthetic.to_bf16(synthetic.outlier_activations(g, n, d, 1.5))
    B = synthetic.to_bf16(synthetic.gaussian_weight(g, d, m))
    parity_linear(A, B, rho)


def test_linear_decode_deterministic():
    A, _ = synthetic.decode_gemv(8, weight=False)
    Ad, Wd = A.cuda(), decode_weight().cuda()
    a = rmm.linear(Ad, Wd, 0.7, return_idx=True)
    b = rmm.linear(Ad, Wd, 0.7, return_idx=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("n,d,m,k", [(4096, 4096, 14336, 2048), (300, 2056, 520, 1000), (257, 1000, 300, 1),
                                     (512, 14336, 4096, 12903), (1000, 777, 136, 700), (129, 64, 8, 64)])
def test_gemm_gathered_matches_the_packed_product(n, d, m, k):
    """The gathered product against the packed one (bit for bit) and against the fp32
    reference: ragged n, m and k, m not a multiple of 8 (partial 16-byte rows), a
    single kept row, narrow last-wave pieces, unsorted-free ascending sets."""
    g = synthetic.rng(n + d + m + k)
    ldp = (k + 7) // 8 * 8
    A = torch.zeros((n, ldp), dtype=torch.bfloat16)
    A[:, :k] = synthetic.to_bf16(g.standard_normal((n, k), dtype=np.float32))
    ldb = (m + 7) // 8 * 8
    Bfull = torch.zeros((d, ldb), dtype=torch.bfloat16)
    Bfull[:, :m] = synthetic.to_bf16(g.standard_normal((d, m), dtype=np.float32) / np.float32(np.sqrt(k)))
    idx = torch.as_tensor(np.sort(g.choice(d, size=k, replace=False)), dtype=torch.int32)
    A, Bd, idx = A.cuda(), Bfull.cuda()[:, :m], idx.cuda()

    def out():  # the library's rule: output rows start 16-byte aligned
        return torch.zeros((n, ldb), dtype=torch.bfloat16, device="cuda")[:, :m]
    Yg = rmm.gemm_gathered(A, k, Bd, idx, out=out())
    bp = rmm.gather_rows(Bd, idx)
    Yp = rmm.gemm_packed(A, k, bp, m, out=out())
    Yg2 = rmm.gemm_gathered(A, k, Bd, idx, out=out())
    torch.cuda.synchronize()
    assert torch.equal(Yg, Yg2), "not deterministic"
    if n > 128:
        assert torch.equal(Yg, Yp), "gathered and packed products differ"
    ref = (A[:, :k].float() @ Bd.float()[idx.long()]).cpu().numpy()
    check_close(Yg.float().cpu().numpy(), ref, f"gathered product n={n} d={d} m={m} k={k}")
