"""The allocation-free selection entry point, rmm_select_noalloc.

Some callers cannot allocate device memory (their framework's allocator owns
it, or a cudaMalloc that may synchronise the device is not acceptable on their
path), so the library offers one selection entry point whose scratch is a fixed
array inside the library.  This test calls it through the C ABI and checks, on
two calls in a row, that it returns exactly what rmm_select returns on the same
inputs.  It lives in its own file, collected last, and needs no state from the
other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")

MAX_SCORES = 262144
UNSUPPORTED = 2


def noalloc_fn():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    L = rmm.lib()
    fn = L.rmm_select_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return L, fn


CASES = [
    # (batch, n, d, causal, rho)
    (1, 4096, 4096, 0, 0.5),      # prefill projection activations
    (32, 512, 128, 0, 0.7),       # per-head query feature selection
    (2, 300, 520, 1, 0.8),        # causal attention probabilities
    (1, 1, 12, 0, 0.5),           # tiny, ragged
    (8, 64, 32768, 0, 0.9),       # exactly the scratch limit
]


def make_input(batch, n, d, causal):
    g = synthetic.rng(900 + batch * 13 + n + d)
    if causal:
        x = [synthetic.causal_softmax_rows(2.0 * g.standard_normal((n, d), dtype=np.float32), d - n)
             for _ in range(batch)]
        A = synthetic.to_bf16(np.stack(x))
    else:
        A = synthetic.to_bf16(synthetic.outlier_activations(g, batch * n, d, 1.5)).reshape(batch, n, d)
    ld = (d + 7) // 8 * 8
    buf = torch.zeros((batch, n, ld), dtype=torch.bfloat16, device="cuda")
    buf[:, :, :d].copy_(A)
    return buf[:, :, :d]


@pytest.mark.parametrize("batch,n,d,causal,rho", CASES)
def test_select_noalloc_matches_select_on_two_calls(batch, n, d, causal, rho):
    L, fn = noalloc_fn()
    A = make_input(batch, n, d, causal)
    idx_ref, _, ret_ref = rmm.select(A, rho, causal=bool(causal))
    k = idx_ref.shape[-1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((batch, k), -1, dtype=torch.int32, device="cuda")
        ret = torch.full((batch,), -1.0, dtype=torch.float64, device="cuda")
        st = fn(A.data_ptr(), batch, A.stride(0), n, d, A.stride(1), causal, rho, idx.data_ptr(), ret.data_ptr(),
                stream)
        assert st == 0, L.rmm_last_error()
        torch.cuda.synchronize()
        assert torch.equal(idx.view_as(idx_ref), idx_ref), f"index sets differ on call {call}"
        assert torch.allclose(ret.view_as(ret_ref), ret_ref, rtol=1e-12, atol=0), f"retained energy, call {call}"
    assert rmm.device_error() == 0


def test_select_noalloc_rejects_sizes_beyond_its_scratch():
    L, fn = noalloc_fn()
    A = torch.zeros((9, 8, 32768), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((9, 16384), dtype=torch.int32, device="cuda")
    st = fn(A.data_ptr(), 9, A.stride(0), 8, 32768, 32768, 0, 0.5, idx.data_ptr(), None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == UNSUPPORTED
    assert str(MAX_SCORES).encode() in L.rmm_last_error()


def test_select_noalloc_back_to_back_calls_with_different_inputs():
    """Two calls on one stream with no synchronisation between them, on inputs whose
    top-k columns differ (the second input's column scales are reversed).  Both
    calls share the scratch array, so the second call's column-score kernel must
    not overwrite scores the first call's selection is still reading: each call's
    index set must equal rmm_select's on its own input."""
    L, fn = noalloc_fn()
    g = synthetic.rng(4242)
    n, d, rho = 512, 4096, 0.5
    base = synthetic.outlier_activations(g, n, d, 1.5)
    A1 = synthetic.to_bf16(base).cuda()
    A2 = synthetic.to_bf16(base[:, ::-1].copy()).cuda()  # column j of A2 is column d-1-j of A1
    ref1, _, _ = rmm.select(A1, rho)
    ref2, _, _ = rmm.select(A2, rho)
    torch.cuda.synchronize()
    assert not torch.equal(ref1, ref2)
    k = ref1.numel()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = [torch.full((k,), -1, dtype=torch.int32, device="cuda") for _ in range(4)]
    for i, A in enumerate((A1, A2, A1, A2)):
        st = fn(A.data_ptr(), 1, n * d, n, d, d, 0, rho, out[i].data_ptr(), None, stream)
        assert st == 0, L.rmm_last_error()
    torch.cuda.synchronize()
    for i, ref in enumerate((ref1, ref2, ref1, ref2)):
        assert torch.equal(out[i], ref), f"call {i} returned another input's index set"
    assert rmm.device_error() == 0
