"""GPU tests of device code that no product call exposes on its own, through the
library's test hooks (declared in include/rmm.h):

* the fused attention's FMA-pipe 2^x (x rounded to the nearest integer n, a
  cubic fitted to 2^f on [-1/2, 1/2], evaluated on packed fp32 pairs) against
  float64 2^x and CUDA's exp2f, at the relative errors it states: 7.6e-5 on
  [-125, 0], 1.6e-4 on [-126, -125) (where the exponent add can produce a
  subnormal), about 2^-126 below -126;
* the timeout path of a bounded wait: the one-CTA tensor-core product with its
  producer's waits made to expire must return, leave code 1 (producer timeout)
  in the device error word, clear it on the read, and leave the context usable
  for a following product that passes parity.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic
from parity import check_close

pytestmark = pytest.mark.gpu

rmm = pytest.importorskip("input_adaptive_reduced_colnorm_b200")

POLY_REL_BOUND = 7.6e-5  # stated bound on [-125, 0]: 7.49e-5 for the exact cubic, plus fp32 rounding
POLY_EDGE_BOUND = 1.6e-4  # on [-126, -125): the result can be subnormal where n = -126
TIMEOUT_PRODUCER = 1


def hooks():
    from input_adaptive_reduced_colnorm_b200 import build
    build.build()
    L = rmm.lib()
    L.rmm_debug_exp2_poly.restype = ctypes.c_int
    L.rmm_debug_exp2_poly.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p]
    L.rmm_debug_gemm_expire_producer.restype = ctypes.c_int
    L.rmm_debug_gemm_expire_producer.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                                 ctypes.c_int64, ctypes.c_void_p]
    return L


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_exp2_cubic_within_its_stated_relative_error():
    L = hooks()
    g = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 0.0, 2_000_001),                  # dense grid
        -np.arange(127, dtype=np.float64),                    # integers: f = 0
        -np.arange(126, dtype=np.float64) - 0.999999,         # n just below an integer
        -np.arange(126, dtype=np.float64) - 0.5,              # ties: f = +-1/2
        -np.arange(126, dtype=np.float64) - 0.499999,         # f just above -1/2
        g.uniform(-126.0, 0.0, 1_000_000),
    ]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yp = torch.empty_like(xd)
    ye = torch.empty_like(xd)
    assert L.rmm_debug_exp2_poly(xd.data_ptr(), yp.data_ptr(), ye.data_ptr(), x.size, stream()) == 0
    torch.cuda.synchronize()
    ref = np.exp2(x.astype(np.float64))
    poly = yp.cpu().numpy().astype(np.float64)
    cuda = ye.cpu().numpy().astype(np.float64)
    rel = np.abs(poly - ref) / ref
    normal = x >= -125.0
    assert rel[normal].max() <= POLY_REL_BOUND, \
        f"max relative error {rel[normal].max():.3e} at x = {x[normal][np.argmax(rel[normal])]}"
    assert rel[~normal].max() <= POLY_EDGE_BOUND
    # CUDA's exp2f is far tighter than the fit; against it the fit keeps its bound
    assert np.max(np.abs(cuda[normal] - ref[normal]) / ref[normal]) < 1e-6
    assert np.max(np.abs(poly[normal] - cuda[normal]) / cuda[normal]) <= POLY_REL_BOUND + 1e-6
    # the largest weights: 2^0 is within the bound of 1, and the fit never exceeds 1 there
    assert abs(poly[x == 0.0][0] - 1.0) <= POLY_REL_BOUND and poly[x == 0.0][0] <= 1.0
    # below -126 the argument is clamped: about 2^-126, never larger than 2^-125
    xs = torch.tensor([-127.0, -150.0, -1e4, float("-inf")], dtype=torch.float32, device="cuda")
    ys, ye2 = torch.empty_like(xs), torch.empty_like(xs)
    assert L.rmm_debug_exp2_poly(xs.data_ptr(), ys.data_ptr(), ye2.data_ptr(), 4, stream()) == 0
    torch.cuda.synchronize()
    assert torch.all(ys.cpu() <= 2.0 ** -125) and torch.all(ys.cpu() >= 0)


def test_expired_producer_wait_returns_records_the_code_and_leaves_the_context_usable():
    L = hooks()
    assert rmm.device_error() == 0  # nothing left over from earlier tests
    g = synthetic.rng(808)
    n, k, m = 128, 1024, 512
    A = synthetic.to_bf16(g.standard_normal((n, k), dtype=np.float32)).cuda()
    B = synthetic.to_bf16(g.standard_normal((k, m), dtype=np.float32) / np.float32(32.0)).cuda()
    Y = torch.zeros((n, m), dtype=torch.bfloat16, device="cuda")
    st = L.rmm_debug_gemm_expire_producer(A.data_ptr(), n, k, k, B.data_ptr(), m, m, Y.data_ptr(), m, stream())
    assert st == 0, L.rmm_last_error()
    torch.cuda.synchronize()  # the kernel returned
    assert rmm.device_error() == TIMEOUT_PRODUCER
    assert rmm.device_error() == 0  # the read cleared it
    # the same product without the hook: correct, and no code recorded
    Y2 = rmm.gemm_packed(A, k, B, m)
    torch.cuda.synchronize()
    check_close(Y2.float().cpu().numpy(), (A.float() @ B.float()).cpu().numpy(), "product after a timeout")
    assert rmm.device_error() == 0
