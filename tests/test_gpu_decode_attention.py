"""GPU parity of decode attention against a key/value cache (rmm_decode_qk,
rmm_decode_pv): one index set per key/value group, chosen on the group's query
rows; the cache rows outside it are never read."""
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


def decode_qk_parity(Q, Kt, rho, nk, scale=1.0, groups=None):
    S, idx = rmm.decode_qk(Q.cuda(), Kt.cuda(), rho, nk=nk, scale=scale, return_idx=True)
    torch.cuda.synchronize()
    Qw = synthetic.widen(Q)
    B, hq, dh = Q.shape
    hkv = Kt.shape[1]
    G = hq // hkv
    k = oracle.retention_count(rho, dh)
    Sc = S.cpu().numpy()
    for b in range(B):
        for g in range(hkv):
            if groups is not None and (b, g) not in groups:
                continue
            A = Qw[b, g * G:(g + 1) * G]
            I = idx[b, g].cpu().numpy().astype(np.int64)
            check_index_set(I, oracle.column_sq_norms(A), k, f"decode qk rho={rho} group {b}/{g}")
            ref = scale * oracle.reduced_product(A, synthetic.widen(Kt[b, g, :, :nk]), I)
            check_close(Sc[b, g * G:(g + 1) * G, :nk], ref, f"decode qk group {b}/{g}")
    return S, idx


def decode_pv_parity(P, V, rho, nk, groups=None):
    O, idx = rmm.decode_pv(P.cuda() if not P.is_cuda else P, V.cuda() if not V.is_cuda else V, rho, nk=nk,
                           return_idx=True)
    torch.cuda.synchronize()
    B, hq, _ = P.shape
    hkv, dh = V.shape[1], V.shape[3]
    G = hq // hkv
    k = oracle.retention_count(rho, nk)
    Oc = synthetic.widen(O.cpu())
    for b in range(B):
        for g in range(hkv):
            if groups is not None and (b, g) not in groups:
                continue
            A = synthetic.widen(P[b, g * G:(g + 1) * G, :nk].cpu())
            I = idx[b, g].cpu().numpy().astype(np.int64)
            check_index_set(I, oracle.column_sq_norms(A), k, f"decode pv rho={rho} group {b}/{g}")
            ref = oracle.reduced_product(A, synthetic.widen(V[b, g, :nk].cpu()), I)
            check_close(Oc[b, g * G:(g + 1) * G], ref, f"decode pv group {b}/{g}")
    return O, idx


@pytest.mark.parametrize("rho", [0.5, 0.7, 1.0])
@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4), (8, 4), (16, 2)])
def test_decode_qk_small(rho, hq, hkv):
    Q, Kt, _, _ = synthetic.decode_attention_inputs(hq=hq, hkv=hkv, nk=1001)
    decode_qk_parity(Q, Kt, rho, 1001, scale=0.088)


@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
@pytest.mark.parametrize("hq,hkv,dh", [(8, 2, 128), (4, 4, 64), (8, 4, 256), (16, 2, 128)])
def test_decode_pv_small(rho, hq, hkv, dh):
    _, _, P, V = synthetic.decode_attention_inputs(hq=hq, hkv=hkv, dh=dh, nk=1001)
    decode_pv_parity(P, V, rho, 1001)


def test_decode_matches_oracle_entry_points_and_repeats():
    Q, Kt, P, V = synthetic.decode_attention_inputs(batch=1, hq=4, hkv=1, dh=64, nk=333)
    S1, I1 = rmm.decode_qk(Q.cuda(), Kt.cuda(), 0.5, nk=333, return_idx=True)
    S2 = rmm.decode_qk(Q.cuda(), Kt.cuda(), 0.5, nk=333)
    O1, J1 = rmm.decode_pv(P.cuda(), V.cuda(), 0.5, nk=333, return_idx=True)
    O2 = rmm.decode_pv(P.cuda(), V.cuda(), 0.5, nk=333)
    torch.cuda.synchronize()
    assert torch.equal(S1, S2) and torch.equal(O1, O2)
    rq = oracle.rmm_decode_qk(synthetic.widen(Q), synthetic.widen(Kt), 0.5, nk=333)
    rp = oracle.rmm_decode_pv(synthetic.widen(P), synthetic.widen(V), 0.5, nk=333)
    assert np.array_equal(I1.cpu().numpy(), rq["I"])
    check_close(S1.cpu().numpy(), rq["S"], "decode qk entry point")
    # the output on the library's own index set, whatever the near-tie band holds ...
    A = synthetic.widen(P[0, :, :333])
    J = J1[0, 0].cpu().numpy().astype(np.int64)
    check_index_set(J, oracle.column_sq_norms(A), oracle.retention_count(0.5, 333), "decode pv entry point")
    check_close(synthetic.widen(O1.cpu())[0], oracle.reduced_product(A, synthetic.widen(V[0, 0, :333]), J),
                "decode pv on the library's set")
    # ... and the oracle's entry point as a whole (its set equals the library's here)
    assert np.array_equal(J1.cpu().numpy(), rp["I"])
    check_close(synthetic.widen(O1.cpu()), rp["O"], "decode pv entry point")


def test_decode_cache_past_nk_is_not_read():
    """Garbage in the cache beyond nk (and NaN in the padding columns of the
    dim-major key cache) must not reach the results."""
    Q, Kt, P, V = synthetic.decode_attention_inputs(batch=1, hq=8, hkv=2, nk=997, L=1024)
    Kt[..., 997:] = float("nan")
    V[:, :, 997:] = float("nan")
    P[..., 997:] = 1.0
    S, _ = decode_qk_parity(Q, Kt, 0.5, 997)
    O, _ = decode_pv_parity(P, V, 0.5, 997)
    assert torch.isfinite(S[..., :997]).all() and torch.isfinite(O).all()


@pytest.mark.parametrize("rho", [0.5, 1.0])
def test_decode_full_context_sampled(rho):
    """Llama-3.1-8B decode shape: 8 sequences x 32 query / 8 key-value heads, head
    dim 128, 32768 cached tokens; a sample of groups checked against the oracle."""
    Q, Kt, P, V = synthetic.decode_attention_inputs_device("cuda")
    groups = {(0, 0), (3, 5), (7, 7)}
    decode_qk_parity(Q.cpu(), Kt.cpu(), rho, 32768, scale=0.088, groups=groups)
    decode_pv_parity(P, V, rho, 32768, groups=groups)
    del Q, Kt, P, V
    torch.cuda.empty_cache()
