"""rmm_linear captured in a CUDA graph: a replay recomputes the scores, the index set
and the product from the buffers' current contents, bit-identical to an eager call.

Launch-bound shapes (a 128 x 1024 x 1024 layer, decode) are meant to run this way:
the graph launches the call's kernels (column scores, selection, packs, product,
fix-up; programmatically chained, clusters included) without per-kernel host work.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity import check_index_set

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")


@pytest.fixture(scope="module", autouse=True)
def built():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    yield
    assert rmm.device_error() == 0


def _inputs(case, seed):
    if case == "linear_128x1024x1024":
        return synthetic.linear_small(seed=seed)
    if case == "decode_n8":
        A, _ = synthetic.decode_gemv(8, seed=seed, d=8192, m=4096, weight=False)
        g = synthetic.rng(seed + 1)
        return A, synthetic.to_bf16(synthetic.gaussian_weight(g, 8192, 4096))
    if case == "prefill_256x1024x2048":
        A, B = synthetic.linear_small(seed=seed, n=256, d=1024, m=2048)
        return A, B
    raise ValueError(case)


@pytest.mark.parametrize("case,rho", [
    ("linear_128x1024x1024", 0.5),
    ("linear_128x1024x1024", 1.0),
    ("decode_n8", 0.5),
    ("prefill_256x1024x2048", 0.7),
])
def test_linear_replays_from_a_cuda_graph(case, rho):
    dev = torch.device("cuda:0")
    A0, B = _inputs(case, 11)
    A1, _ = _inputs(case, 12)  # another activation matrix: another index set
    Ad = A0.to(dev).contiguous()
    Bd = B.to(dev).contiguous()
    n, d = Ad.shape
    m = Bd.shape[1]
    Y = torch.empty((n, m), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(rmm.lib().rmm_linear_workspace_bytes(n, d, m, float(rho)), 256), dtype=torch.uint8,
                     device=dev)

    # eager references on both inputs
    Y_e0, I_e0 = rmm.linear(Ad, Bd, rho, return_idx=True)
    Y_e1, I_e1 = rmm.linear(A1.to(dev), Bd, rho, return_idx=True)
    torch.cuda.synchronize()

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(2):
            rmm.linear(Ad, Bd, rho, out=Y, workspace=ws)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        _, I_g = rmm.linear(Ad, Bd, rho, out=Y, return_idx=True, workspace=ws)

    for A_now, Y_ref, I_ref in ((A0, Y_e0, I_e0), (A1, Y_e1, I_e1), (A0, Y_e0, I_e0)):
        Ad.copy_(A_now.to(dev))
        Y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(I_g, I_ref), f"{case} rho={rho}: replayed index set differs from the eager call"
        assert torch.equal(Y, Y_ref), f"{case} rho={rho}: replayed product differs from the eager call"

    # the replayed index set is the oracle's (near ties logged by the helper)
    q = oracle.column_sq_norms(synthetic.widen(A0))
    k = oracle.retention_count(rho, d)
    Ad.copy_(A0.to(dev))
    g.replay()
    torch.cuda.synchronize()
    check_index_set(I_g.cpu().numpy().astype(np.int64), q, k, f"graph {case} rho={rho}")
    del g
