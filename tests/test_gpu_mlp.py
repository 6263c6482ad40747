"""GPU parity of the MLP block (rmm_mlp): one index set on X shared by gate and up,
the fused tensor-core product writing H = SiLU(gate) * up, and the down projection
as RMM on H with its own rho.

Stage by stage: the gate / up index set is compared with the oracle's on X; H
with oracle.mlp_gate_up_rows on the GPU's index set; the down projection with
the oracle's RMM on the GPU's own H (H is bf16, so its column norms, and with
them the down selection, are those of the rounded H)."""
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


def mlp_parity(X, Wg, Wu, Wd, rho_gu, rho_down, rows=None):
    Xd, Wgd, Wud, Wdd = X.cuda(), Wg.cuda(), Wu.cuda(), Wd.cuda()
    Y, H, i_gu, i_dn = rmm.mlp(Xd, Wgd, Wud, Wdd, rho_gu, rho_down, return_idx=True)
    torch.cuda.synchronize()
    n, d = X.shape
    f = Wg.shape[1]
    Xw = synthetic.widen(X)
    I = i_gu.cpu().numpy().astype(np.int64)
    check_index_set(I, oracle.column_sq_norms(Xw), oracle.retention_count(rho_gu, d),
                    f"mlp gate/up n={n} d={d} rho={rho_gu}")
    r = np.arange(n) if rows is None else np.asarray(rows)
    Hw = synthetic.widen(H.cpu())
    check_close(Hw[r], oracle.mlp_gate_up_rows(Xw, synthetic.widen(Wg), synthetic.widen(Wu), I, r), "mlp H")
    J = i_dn.cpu().numpy().astype(np.int64)
    check_index_set(J, oracle.column_sq_norms(Hw), oracle.retention_count(rho_down, f),
                    f"mlp down n={n} f={f} rho={rho_down}")
    check_close(synthetic.widen(Y.cpu())[r], oracle.rmm_linear_rows(Hw, synthetic.widen(Wd), J, r), "mlp Y")
    return Y, H


@pytest.mark.parametrize("rho_gu,rho_down", [(0.5, 0.5), (0.8, 0.5), (1.0, 1.0), (0.7, 1.0)])
def test_mlp_small_ragged(rho_gu, rho_down):
    """n, d, f, m off every tile size (f = 392: the last 128-column tile is ragged)."""
    X, Wg, Wu, Wd = synthetic.mlp_block(n=300, d=520, f=392, m=264)
    mlp_parity(X, Wg, Wu, Wd, rho_gu, rho_down)


def test_mlp_matches_the_oracle_entry_point_and_repeats():
    X, Wg, Wu, Wd = synthetic.mlp_block(n=160, d=256, f=512, m=128)
    Xd, Wgd, Wud, Wdd = X.cuda(), Wg.cuda(), Wu.cuda(), Wd.cuda()
    Y1, H1, i1, j1 = rmm.mlp(Xd, Wgd, Wud, Wdd, 0.5, 0.5, return_idx=True)
    Y2 = rmm.mlp(Xd, Wgd, Wud, Wdd, 0.5, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    ref = oracle.rmm_mlp_gate_up(synthetic.widen(X), synthetic.widen(Wg), synthetic.widen(Wu), 0.5)
    assert np.array_equal(i1.cpu().numpy(), ref["I"])
    check_close(synthetic.widen(H1.cpu()), ref["H"], "mlp H entry point")


def test_mlp_identity_weights_keep_the_same_columns():
    """Wg = Wu = I: H = SiLU(x) x on the kept columns of X and exactly 0 elsewhere,
    so gate and up both read the shared index set."""
    g = synthetic.rng(36)
    X = synthetic.to_bf16(synthetic.outlier_activations(g, 256, 256, 1.0))
    eye = torch.eye(256, dtype=torch.bfloat16)
    Wd = synthetic.to_bf16(synthetic.gaussian_weight(g, 256, 64))
    Y, H, i_gu, _ = rmm.mlp(X.cuda(), eye.cuda(), eye.cuda(), Wd.cuda(), 0.5, 1.0, return_idx=True)
    torch.cuda.synchronize()
    keep = np.zeros(256, dtype=bool)
    keep[i_gu.cpu().numpy()] = True
    Hw = synthetic.widen(H.cpu())
    assert not Hw[:, ~keep].any()
    x = synthetic.widen(X)[:, keep]
    check_close(Hw[:, keep], x * x / (1.0 + np.exp(-x)), "identity gate/up")


@pytest.mark.parametrize("rho_gu,rho_down", [(0.5, 0.5), (0.8, 0.5)])
def test_mlp_llama8b_sampled(rho_gu, rho_down):
    """Llama-3.1-8B MLP block at n = 4096 tokens (d = 4096, f = 14336); a row sample
    is checked against the oracle."""
    X, Wg, Wu, Wd = synthetic.mlp_block()
    rows = np.concatenate([np.arange(0, 4096, 331), [4095]])
    mlp_parity(X, Wg, Wu, Wd, rho_gu, rho_down, rows=rows)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [1, 8, 32])
def test_mlp_decode_rows(n):
    """Decode-sized blocks (n <= 32): short-matrix column scores, the down
    projection on the decode product; H and Y checked as for any n."""
    X, Wg, Wu, Wd = synthetic.mlp_block(n=n, d=1040, f=776, m=264)
    mlp_parity(X, Wg, Wu, Wd, 0.5, 0.5)
    mlp_parity(X, Wg, Wu, Wd, 0.7, 1.0)
