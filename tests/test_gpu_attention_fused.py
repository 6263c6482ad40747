"""GPU parity of the fused attention with a reduced score product (rmm_attention):
per query head, the index set of rmm_qk, then softmax(scale Q_I K_I^T) V with S
and P kept on chip.  References: the oracle's TopK for the index sets (near-tie
band logged) and oracle.attention_rows on the library's own set for the output."""
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


def check_heads(O, idx, Q, K, V, rho, causal, scale, rows=None):
    B, hq, nq, dh = Q.shape
    hkv = K.shape[1]
    k = oracle.retention_count(rho, dh)
    r = np.arange(nq) if rows is None else np.asarray(rows)
    rsel = torch.as_tensor(r, device=O.device)
    for b in range(B):
        for h in range(hq):
            Qh = synthetic.widen(Q[b, h])
            g = oracle.kv_head(h, hq, hkv)
            I = idx[b, h].cpu().numpy().astype(np.int64)
            check_index_set(I, oracle.column_sq_norms(Qh), k, f"fused attention rho={rho} head {b}/{h}")
            ref = oracle.attention_rows(Qh, synthetic.widen(K[b, g]), synthetic.widen(V[b, g]), I, r, causal, scale)
            check_close(synthetic.widen(O[b, h][rsel].cpu()), ref, f"fused attention head {h}")


def fused_parity(Q, K, V, rho, causal, scale, rows=None):
    O, idx = rmm.attention(Q.cuda(), K.cuda(), V.cuda(), rho, causal=causal, scale=scale, return_idx=True)
    torch.cuda.synchronize()
    check_heads(O, idx, Q, K, V, rho, causal, scale, rows)
    return O, idx


def qkv(hq, hkv, nq, nk, seed=40, batch=1):
    g = synthetic.rng(seed)
    Q = synthetic.to_bf16(g.standard_normal((batch, hq, nq, 128), dtype=np.float32) * np.exp(g.standard_normal(128)).astype(np.float32))
    K = synthetic.to_bf16(g.standard_normal((batch, hkv, nk, 128), dtype=np.float32))
    V = synthetic.to_bf16(g.standard_normal((batch, hkv, nk, 128), dtype=np.float32))
    return Q, K, V


@pytest.mark.parametrize("rho", [0.3, 0.5, 0.7, 1.0])
@pytest.mark.parametrize("causal", [True, False])
def test_fused_attention_small_gqa(rho, causal):
    """4 query / 2 key-value heads, 300 rows (ragged last query tile and key block)."""
    Q, K, V = qkv(4, 2, 300, 300)
    fused_parity(Q, K, V, rho, causal, 0.088)


@pytest.mark.parametrize("rho", [0.4, 0.8, 1.0])
def test_fused_attention_batch_of_two(rho):
    """Two batch items of 4 query / 2 key-value heads (different data per item):
    the item index of Q, K, V and O, the packed operands (rho 0.4) and the zeroed
    Q (rho 0.8) per item."""
    Q, K, V = qkv(4, 2, 260, 260, seed=47, batch=2)
    fused_parity(Q, K, V, rho, True, 0.09)


def test_fused_attention_rectangular_causal():
    """nq < nk: bottom-right alignment, several key blocks per query tile."""
    Q, K, V = qkv(2, 1, 200, 520, seed=41)
    fused_parity(Q, K, V, 0.5, True, 0.088)


def test_fused_attention_matches_oracle_and_repeats():
    Q, K, V = qkv(2, 1, 256, 256, seed=42)
    O1, I1 = rmm.attention(Q.cuda(), K.cuda(), V.cuda(), 0.5, scale=0.1, return_idx=True)
    O2 = rmm.attention(Q.cuda(), K.cuda(), V.cuda(), 0.5, scale=0.1)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)
    ref = oracle.rmm_attention(synthetic.widen(Q), synthetic.widen(K), synthetic.widen(V), 0.5, causal=True, scale=0.1)
    assert np.array_equal(I1.cpu().numpy(), ref["I"])
    check_close(synthetic.widen(O1.cpu()), ref["O"], "fused attention entry point")


def test_fused_attention_gqa_seq4096_all_heads():
    """32 query / 8 key-value heads, seq 4096, causal, rho = 0.7 and 0.5: the GPU's
    fp64 column scores and index sets of all 32 heads, and a row sample of every
    head's output."""
    Q, K = synthetic.qk_inputs()
    V = synthetic.to_bf16(synthetic.rng(43).standard_normal((1, 8, 4096, 128), dtype=np.float32))
    _, cs, _ = rmm.select(Q[0].cuda(), 0.5)
    torch.cuda.synchronize()
    for h in range(32):
        check_colsq(cs[h].cpu().numpy(), oracle.column_sq_norms(synthetic.widen(Q[0, h])))
    rows = np.concatenate([np.arange(0, 4096, 397), [4095]])
    for rho in (0.7, 0.5):
        fused_parity(Q, K, V, rho, True, 0.088, rows=rows)
