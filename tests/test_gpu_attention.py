"""GPU parity of the attention-side reductions: rmm_qk (head-dim selection on Q,
K gathered under GQA, causal -inf scores) and rmm_pv (token-position selection
on P, V rows gathered).

Every reference below is an oracle function: the index sets against the oracle's
TopK of its own fp64 scores (near-tie band logged), the products against
oracle.qk_scores_rows / oracle.pv_output_rows on the library's own index set."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check_close, check_colsq, check_index_set

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")


@pytest.fixture(scope="module", autouse=True)
def built():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    yield
    assert rmm.device_error() == 0


def check_qk_heads(S, idx, Q, K, rho, causal, scale, rows=None):
    """Every head: index set vs the oracle's, sampled (or all) rows of S vs
    oracle.qk_scores_rows on the library's set."""
    Qw, Kw = synthetic.widen(Q), synthetic.widen(K)
    b_, hq, nq, dh = Q.shape
    hkv = K.shape[1]
    k = oracle.retention_count(rho, dh)
    r = np.arange(nq) if rows is None else np.asarray(rows)
    rsel = torch.as_tensor(r, device=S.device)
    for b in range(b_):
        for h in range(hq):
            I = idx[b, h].cpu().numpy().astype(np.int64)
            check_index_set(I, oracle.column_sq_norms(Qw[b, h]), k, f"qk rho={rho} head {b}/{h}")
            ref = oracle.qk_scores_rows(Qw[b, h], Kw[b, oracle.kv_head(h, hq, hkv)], I, r, causal, scale)
            check_close(S[b, h][rsel].cpu().numpy(), ref, f"qk head {h}")


def qk_parity(Q, K, rho, causal, scale=1.0, rows=None):
    S, idx = rmm.qk(Q.cuda(), K.cuda(), rho, causal=causal, scale=scale, return_idx=True)
    torch.cuda.synchronize()
    check_qk_heads(S, idx, Q, K, rho, causal, scale, rows)
    return S, idx


@pytest.mark.parametrize("rho", [0.5, 0.7, 1.0])
@pytest.mark.parametrize("causal", [True, False])
def test_qk_small_gqa(rho, causal):
    Q, K = synthetic.qk_inputs(hq=4, hkv=2, n=300)
    qk_parity(Q, K, rho, causal, scale=0.125)


def test_qk_matches_oracle_entry_point():
    Q, K = synthetic.qk_inputs(hq=4, hkv=1, n=136)
    S, idx = rmm.qk(Q.cuda(), K.cuda(), 0.5, causal=True, return_idx=True)
    torch.cuda.synchronize()
    ref = oracle.rmm_qk(synthetic.widen(Q), synthetic.widen(K), 0.5, causal=True)
    assert np.array_equal(idx.cpu().numpy(), ref["I"])
    check_close(S.cpu().numpy(), ref["S"], "qk entry point")


def test_qk_rectangular_causal_alignment():
    g = synthetic.rng(41)
    Q = synthetic.to_bf16(g.standard_normal((1, 2, 100, 128), dtype=np.float32))
    K = synthetic.to_bf16(g.standard_normal((1, 1, 264, 128), dtype=np.float32))
    qk_parity(Q, K, 0.5, True)


def test_qk_gqa_seq4096_all_heads():
    """32 query heads / 8 key-value heads, head_dim 128, seq 4096, causal fp32 scores
    at rho = 0.7 and 0.5: the GPU's fp64 column scores of all 32 heads against the
    oracle's, every head's index set, and a row sample of every head's scores."""
    Q, K = synthetic.qk_inputs()
    Qd, Kd = Q.cuda(), K.cuda()
    _, cs, _ = rmm.select(Qd[0], 0.5)  # the selection kernels rmm_qk runs, batched over heads
    torch.cuda.synchronize()
    Qw = synthetic.widen(Q)
    for h in range(Q.shape[1]):
        check_colsq(cs[h].cpu().numpy(), oracle.column_sq_norms(Qw[0, h]))
    rows = np.concatenate([np.arange(0, 4096, 257), [4095]])
    for rho in (0.7, 0.5):
        S, idx = rmm.qk(Qd, Kd, rho, causal=True, return_idx=True)
        torch.cuda.synchronize()
        check_qk_heads(S, idx, Q, K, rho, True, 1.0, rows)
        del S
    torch.cuda.empty_cache()


def check_pv_heads(O, idx, P, V, rho, causal, rows=None):
    b_, h_, nq, nk = P.shape
    hkv = V.shape[1]
    k = oracle.retention_count(rho, nk)
    r = np.arange(nq) if rows is None else np.asarray(rows)
    rsel = torch.as_tensor(r, device=O.device)
    for b in range(b_):
        for h in range(h_):
            Ph = synthetic.widen(P[b, h])
            Vg = synthetic.widen(V[b, oracle.kv_head(h, h_, hkv)])
            q = oracle.column_sq_norms(Ph, causal=causal)
            I = idx[b, h].cpu().numpy().astype(np.int64)
            check_index_set(I, q, k, f"pv rho={rho} head {b}/{h}")
            ref = oracle.pv_output_rows(Ph, Vg, I, r, causal)
            check_close(synthetic.widen(O[b, h][rsel].cpu()), ref, f"pv head {h}")


def pv_parity(P, V, rho, causal, rows=None):
    O, idx = rmm.pv(P.cuda() if not P.is_cuda else P, V.cuda() if not V.is_cuda else V, rho, causal=causal,
                    return_idx=True)
    torch.cuda.synchronize()
    check_pv_heads(O, idx, P, V, rho, causal, rows)
    return O, idx


@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
@pytest.mark.parametrize("causal", [True, False])
def test_pv_small(rho, causal):
    P, V = synthetic.pv_inputs(heads=2, n=520)
    pv_parity(P, V, rho, causal)


def test_pv_head_dim_64_and_gqa():
    P, V = synthetic.pv_inputs(heads=4, n=264, dh=64, kv_heads=2)
    pv_parity(P, V, 0.5, True)


def test_pv_entry_point_with_junk_above_diagonal():
    """Garbage above the diagonal: index sets against the oracle's causal scores, the
    output against oracle.pv_output_rows on the library's own sets (always), and the
    oracle's entry point as a whole (its own sets equal the library's here)."""
    P, V = synthetic.pv_inputs(heads=2, n=200)
    junk = torch.triu(torch.full((200, 200), 3.0), 1).to(torch.bfloat16)
    Pj = P + junk
    O, idx = rmm.pv(Pj.cuda(), V.cuda(), 0.5, causal=True, return_idx=True)
    torch.cuda.synchronize()
    check_pv_heads(O, idx, Pj, V, 0.5, True)
    ref = oracle.rmm_pv(synthetic.widen(Pj), synthetic.widen(V), 0.5, causal=True)
    assert np.array_equal(idx.cpu().numpy(), ref["I"])
    check_close(synthetic.widen(O.cpu()), ref["O"], "pv entry point")


@pytest.mark.parametrize("rho", [1.0, 0.8])
def test_pv_dense_and_reduced_ignore_entries_above_the_diagonal(rho):
    """Causal PV treats P[i, j] with j > i + (nk - nq) as zero on every path."""
    P, V = synthetic.pv_inputs(heads=2, n=328)
    junk = torch.triu(torch.full((328, 328), 5.0), 1).to(torch.bfloat16)
    pv_parity(P + junk, V, rho, True)


def test_pv_seq16384_all_heads():
    """Long-context PV: 32 heads x 16384 x 16384 causal softmax probabilities drawn on
    the device, rho = 0.8 and 0.5.  All 32 heads: the GPU's fp64 causal column scores
    against the oracle's, the index sets, and a row sample of each head's output
    against oracle.pv_output_rows on the library's set.  Each head is widened once for
    both rho values."""
    P, V = synthetic.pv_inputs_device("cuda", heads=32, n=16384)
    b_, h_, nq, nk = P.shape
    rows = np.concatenate([np.arange(0, 16384, 1031), [16383]])
    rsel = torch.as_tensor(rows, device="cuda")
    runs = {}
    for rho in (0.8, 0.5):
        O, idx = rmm.pv(P, V, rho, causal=True, return_idx=True)
        torch.cuda.synchronize()
        runs[rho] = (synthetic.widen(O[0][:, rsel].cpu()), idx[0].cpu().numpy().astype(np.int64))
        del O
    _, cs, _ = rmm.select(P[0], 0.5, causal=True)
    torch.cuda.synchronize()
    cs = cs.cpu().numpy()
    for h in range(h_):
        Ph = synthetic.widen(P[0, h].cpu())
        Vg = synthetic.widen(V[0, h].cpu())
        q = oracle.column_sq_norms(Ph, causal=True)
        check_colsq(cs[h], q)
        for rho, (Orows, I) in runs.items():
            check_index_set(I[h], q, oracle.retention_count(rho, nk), f"pv seq16384 rho={rho} head {h}")
            check_close(Orows[h], oracle.pv_output_rows(Ph, Vg, I[h], rows, True), f"pv seq16384 head {h}")
        del Ph
    del P, V
    torch.cuda.empty_cache()
