"""GPU parity of the attention-side reductions: rmm_qk (head-dim selection on Q,
K gathered under GQA, causal -inf scores) and rmm_pv (token-position selection
on P, V rows gathered)."""
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


def qk_parity(Q, K, rho, causal, scale=1.0, heads=None, rows=None):
    S, idx = rmm.qk(Q.cuda(), K.cuda(), rho, causal=causal, scale=scale, return_idx=True)
    torch.cuda.synchronize()
    Qw, Kw = synthetic.widen(Q), synthetic.widen(K)
    b_, hq, nq, dh = Q.shape
    hkv = K.shape[1]
    k = oracle.retention_count(rho, dh)
    heads = range(hq) if heads is None else heads
    for b in range(b_):
        for h in heads:
            q = oracle.column_sq_norms(Qw[b, h])
            I = idx[b, h].cpu().numpy().astype(np.int64)
            check_index_set(I, q, k)
            r = np.arange(nq) if rows is None else np.asarray(rows)
            Qh = Qw[b, h][r][:, I]
            Kg = Kw[b, oracle.kv_head(h, hq, hkv)][:, I]
            ref = scale * (Qh @ Kg.T)
            if causal:
                nk = K.shape[2]
                vis = np.minimum(nk, r + (nk - nq) + 1)
                ref[np.arange(nk)[None, :] >= vis[:, None]] = -np.inf
            got = S[b, h][torch.as_tensor(r, device=S.device)].cpu().numpy()
            check_close(got, ref, f"qk head {h}")
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


@pytest.mark.parametrize("rho", [0.5, 0.7])
def test_qk_gqa_seq4096_sampled(rho):
    """32 query heads / 8 key-value heads, head_dim 128, seq 4096, causal fp32 scores."""
    Q, K = synthetic.qk_inputs()
    rows = np.concatenate([np.arange(0, 4096, 257), [4095]])
    qk_parity(Q, K, rho, True, heads=[0, 3, 4, 17, 31], rows=rows)


def pv_parity(P, V, rho, causal, heads=None, rows=None):
    O, idx = rmm.pv(P.cuda() if not P.is_cuda else P, V.cuda() if not V.is_cuda else V, rho, causal=causal,
                    return_idx=True)
    torch.cuda.synchronize()
    b_, h_, nq, nk = P.shape
    hkv = V.shape[1]
    k = oracle.retention_count(rho, nk)
    heads = range(h_) if heads is None else heads
    for b in range(b_):
        for h in heads:
            Ph = synthetic.widen(P[b, h])
            Vg = synthetic.widen(V[b, oracle.kv_head(h, h_, hkv)])
            q = oracle.column_sq_norms(Ph, causal=causal)
            I = idx[b, h].cpu().numpy().astype(np.int64)
            check_index_set(I, q, k)
            r = np.arange(nq) if rows is None else np.asarray(rows)
            Pr = Ph[r][:, I].copy()
            if causal:
                vis = np.minimum(nk, r + (nk - nq) + 1)
                Pr[I[None, :] >= vis[:, None]] = 0.0
            ref = Pr @ Vg[I, :]
            got = synthetic.widen(O[b, h][torch.as_tensor(r, device=O.device)].cpu())
            check_close(got, ref, f"pv head {h}")
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
    P, V = synthetic.pv_inputs(heads=2, n=200)
    junk = torch.triu(torch.full((200, 200), 3.0), 1).to(torch.bfloat16)
    Pj = P + junk
    O, idx = rmm.pv(Pj.cuda(), V.cuda(), 0.5, causal=True, return_idx=True)
    torch.cuda.synchronize()
    ref = oracle.rmm_pv(synthetic.widen(Pj), synthetic.widen(V), 0.5, causal=True)
    for h in range(2):
        q = oracle.column_sq_norms(synthetic.widen(Pj[0, h]), causal=True)
        check_index_set(idx[0, h].cpu().numpy(), q, 100)
    if np.array_equal(idx.cpu().numpy(), ref["I"]):
        check_close(synthetic.widen(O.cpu()), ref["O"], "pv entry point")


@pytest.mark.parametrize("rho", [1.0, 0.8])
def test_pv_dense_and_reduced_ignore_entries_above_the_diagonal(rho):
    """Causal PV treats P[i, j] with j > i + (nk - nq) as zero on every path."""
    P, V = synthetic.pv_inputs(heads=2, n=328)
    junk = torch.triu(torch.full((328, 328), 5.0), 1).to(torch.bfloat16)
    Pj = P + junk
    O, idx = rmm.pv(Pj.cuda(), V.cuda(), rho, causal=True, return_idx=True)
    torch.cuda.synchronize()
    for h in range(2):
        q = oracle.column_sq_norms(synthetic.widen(Pj[0, h]), causal=True)
        I = idx[0, h].cpu().numpy().astype(np.int64)
        check_index_set(I, q, oracle.retention_count(rho, 328))
        Ph = synthetic.widen(Pj[0, h])
        Pr = Ph[:, I].copy()
        Pr[I[None, :] > np.arange(328)[:, None]] = 0.0
        check_close(synthetic.widen(O[0, h].cpu()), Pr @ synthetic.widen(V[0, h])[I, :], f"pv junk head {h}")


@pytest.mark.parametrize("rho", [0.5, 0.8])
def test_pv_seq16384_sampled(rho):
    """Long-context PV: 32 heads x 16384 x 16384 causal softmax probabilities drawn on
    the device; two heads and a row sample are checked against the oracle."""
    P, V = synthetic.pv_inputs_device("cuda", heads=32, n=16384)
    rows = np.concatenate([np.arange(0, 16384, 1031), [16383]])
    pv_parity(P, V, rho, True, heads=[0, 29], rows=rows)
    del P, V
    torch.cuda.empty_cache()
