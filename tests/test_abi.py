"""Host-side checks of the C ABI (no GPU needed).

The library must load and export every function include/rmm.h declares, agree
with the hand-derived k table, and reject bad arguments with the documented
status before touching the device (on a machine without a GPU any device call
would surface as RMM_ERR_CUDA instead, so the exact codes below also show that
nothing was enqueued).
"""
import json
import os
import re

import pytest

import input_adaptive_reduced_colnorm_b200 as rmm
from input_adaptive_reduced_colnorm_b200 import build as rmm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rmm.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA_ERR, TIMEOUT = range(6)
P16 = 0x10000  # a 16-byte aligned fake device address (never dereferenced)
P_MIS = 0x10002


@pytest.fixture(scope="module")
def L():
    rmm_build.build()
    return rmm.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rmm_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"rmm_select", "rmm_linear", "rmm_qk", "rmm_pv", "rmm_k"} <= set(names)
    for name in names:
        assert hasattr(L, name), name
    assert L.rmm_version().startswith(b"rmm-b200")


def test_k_table_matches_hand_fixture(L):
    with open(os.path.join(ROOT, "tests", "golden", "retention_count.json")) as f:
        fx = json.load(f)
    for rho, d, k in fx["cases"]:
        assert L.rmm_k(rho, d) == k, (rho, d)
    for rho, d in fx["invalid"]:
        assert L.rmm_k(float(rho), d) == -1


def test_status_strings(L):
    for s in range(6):
        assert L.rmm_status_string(s)
    assert L.rmm_last_error() is not None


def lin(L, A=P16, n=64, d=128, lda=128, B=P16, m=64, ldb=64, Y=P16, ldy=64, rho=0.5, idx=None, ws=None, wsb=0):
    return L.rmm_linear(A, n, d, lda, B, m, ldb, Y, ldy, rho, idx, ws, wsb, None)


@pytest.mark.parametrize("rho", [0.0, -0.5, 1.0000001, float("nan"), float("inf")])
def test_linear_rejects_bad_rho(L, rho):
    assert lin(L, rho=rho) == INVALID
    assert b"rho" in L.rmm_last_error()


def test_linear_argument_errors(L):
    assert lin(L, A=None) == INVALID
    assert lin(L, Y=None) == INVALID
    assert lin(L, n=0) == INVALID
    assert lin(L, lda=64) == INVALID          # lda < d
    assert lin(L, ldb=32) == INVALID          # ldb < m
    assert lin(L, A=P_MIS) == UNSUPPORTED     # misaligned pointer
    assert lin(L, lda=132) == UNSUPPORTED     # leading dim not a multiple of 8
    need = L.rmm_linear_workspace_bytes(64, 128, 64, 0.5)
    assert need > 0
    assert lin(L, ws=None, wsb=0) == WORKSPACE
    assert lin(L, ws=P16, wsb=need - 1) == WORKSPACE
    assert b"workspace" in L.rmm_last_error()


def test_select_argument_errors(L):
    def sel(A=P16, batch=1, bs=0, n=16, d=64, lda=64, causal=0, rho=0.5, idx=P16, cs=None, rt=None, ws=None, wsb=0):
        return L.rmm_select(A, batch, bs, n, d, lda, causal, rho, idx, cs, rt, ws, wsb, None)
    assert sel(idx=None) == INVALID
    assert sel(rho=2.0) == INVALID
    assert sel(causal=2) == INVALID
    assert sel(batch=2, bs=8) == INVALID           # batch items overlap
    assert sel(d=40000, lda=40000) == UNSUPPORTED  # beyond the documented d limit
    assert sel(lda=68) == UNSUPPORTED
    assert sel(ws=None) == WORKSPACE               # no colsq_out and no workspace


def test_qk_pv_argument_errors(L):
    def qk(Q=P16, K=P16, S=P16, b=1, hq=4, hkv=2, nq=64, nk=64, dh=128, causal=1, scale=1.0, rho=0.5, ws=None,
           wsb=0):
        return L.rmm_qk(Q, K, S, b, hq, hkv, nq, nk, dh, causal, scale, rho, None, ws, wsb, None)
    assert qk(hkv=3) == INVALID          # Hq % Hkv != 0
    assert qk(scale=float("nan")) == INVALID
    assert qk(dh=100) == UNSUPPORTED
    assert qk(nk=66) == UNSUPPORTED
    assert qk() == WORKSPACE

    def pv(P=P16, V=P16, O=P16, b=1, h=4, hkv=4, nq=64, nk=64, dh=128, causal=1, rho=0.5, ws=None, wsb=0):
        return L.rmm_pv(P, V, O, b, h, hkv, nq, nk, dh, causal, rho, None, ws, wsb, None)
    assert pv(hkv=3) == INVALID
    assert pv(O=None) == INVALID
    assert pv(dh=96) == UNSUPPORTED
    assert pv(nk=60) == UNSUPPORTED
    assert pv() == WORKSPACE


def test_workspace_queries(L):
    assert L.rmm_linear_workspace_bytes(4096, 4096, 4096, 1.0) == 0
    a = L.rmm_linear_workspace_bytes(4096, 4096, 4096, 0.5)
    b = L.rmm_linear_workspace_bytes(4096, 4096, 4096, 0.9)
    assert 0 < a < b
    assert a >= 4096 * 2048 * 2
    assert L.rmm_qk_workspace_bytes(1, 32, 8, 4096, 4096, 128, 1.0) == 0
    assert L.rmm_qk_workspace_bytes(1, 32, 8, 4096, 4096, 128, 0.5) >= 2 * 32 * 4096 * 64 * 2
    assert L.rmm_pv_workspace_bytes(1, 32, 32, 1024, 1024, 128, 0.5) >= 32 * 1024 * 128 * 2
    assert L.rmm_select_workspace_bytes(3, 10, 100) >= 3 * 100 * 8


def test_binding_refuses_cpu_tensors():
    """Every public call refuses host tensors before anything reaches the library:
    there is no CPU path."""
    import torch
    bf = torch.bfloat16
    A = torch.zeros((4, 16), dtype=bf)
    B = torch.zeros((16, 8), dtype=bf)
    idx = torch.zeros(8, dtype=torch.int32)
    Q4 = torch.zeros((1, 2, 8, 64), dtype=bf)
    calls = [
        lambda: rmm.linear(A, B, 0.5),
        lambda: rmm.select(A, 0.5),
        lambda: rmm.gather_columns(A, idx),
        lambda: rmm.gather_rows(B, idx),
        lambda: rmm.gemm_packed(A, 16, B, 8),
        lambda: rmm.qk(Q4, Q4, 0.5),
        lambda: rmm.pv(torch.zeros((1, 2, 8, 8), dtype=bf), Q4, 0.5),
        lambda: rmm.attention(Q4, Q4, Q4, 0.5),
        lambda: rmm.linear_int8(A, torch.zeros((16, 8), dtype=torch.int8), torch.ones(8), 0.5),
        lambda: rmm.mlp(A, B, B, torch.zeros((8, 16), dtype=bf), 0.5, 0.5),
        lambda: rmm.decode_qk(torch.zeros((1, 2, 64), dtype=bf), torch.zeros((1, 1, 64, 8), dtype=bf), 0.5),
        lambda: rmm.decode_pv(torch.zeros((1, 2, 8), dtype=bf), torch.zeros((1, 1, 8, 64), dtype=bf), 0.5),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(TypeError, match="CUDA tensor"):
            call()


def test_decode_attention_argument_errors(L):
    def dqk(Q=P16, Kt=P16, S=P16, b=1, hq=8, hkv=2, dh=128, nk=100, ldk=104, lds=100, scale=1.0, rho=0.5, ws=None,
            wsb=0):
        return L.rmm_decode_qk(Q, Kt, S, b, hq, hkv, dh, nk, ldk, lds, scale, rho, None, ws, wsb, None)
    assert dqk(hkv=3) == INVALID             # hq % hkv
    assert dqk(ldk=96) == INVALID            # ldk < nk
    assert dqk(scale=float("inf")) == INVALID
    assert dqk(hq=24, hkv=2) == UNSUPPORTED  # group of 12
    assert dqk(dh=100) == UNSUPPORTED
    assert dqk(ldk=108) == UNSUPPORTED       # not a multiple of 8
    assert dqk(lds=102) == UNSUPPORTED       # not a multiple of 4
    assert dqk() == WORKSPACE
    assert L.rmm_decode_qk_workspace_bytes(1, 8, 2, 128, 1.0) == 0

    def dpv(P=P16, V=P16, O=P16, b=1, hq=8, hkv=2, nk=100, ldp=104, cap=100, dh=128, rho=0.5, ws=None, wsb=0):
        return L.rmm_decode_pv(P, V, O, b, hq, hkv, nk, ldp, cap, dh, rho, None, ws, wsb, None)
    assert dpv(cap=99) == INVALID
    assert dpv(dh=96) == UNSUPPORTED
    assert dpv(hq=16, hkv=2, dh=256) == UNSUPPORTED  # 8 x 256 > 1024
    assert dpv(ldp=100) == UNSUPPORTED
    assert dpv(nk=40000, ldp=40000, cap=40000) == UNSUPPORTED
    assert dpv() == WORKSPACE
    assert L.rmm_decode_pv_workspace_bytes(1, 8, 2, 100, 128, 1.0) > 0  # partial sums even at rho = 1


def test_mlp_argument_errors(L):
    def mlp(X=P16, n=300, d=512, ldx=512, Wg=P16, Wu=P16, f=1024, ldw=1024, Wd=P16, m=512, ldwd=512, H=P16,
            ldh=1024, Y=P16, ldy=512, rg=0.5, rd=0.5, ws=None, wsb=0):
        return L.rmm_mlp(X, n, d, ldx, Wg, Wu, f, ldw, Wd, m, ldwd, H, ldh, Y, ldy, rg, rd, None, None, ws, wsb, None)
    assert mlp(rg=0.0) == INVALID
    assert mlp(rd=1.5) == INVALID
    assert mlp(H=None) == INVALID
    assert mlp(ldh=1000) == INVALID          # ldh < f
    assert mlp(ldw=1028) == UNSUPPORTED
    assert mlp(d=40000, ldx=40000) == UNSUPPORTED
    assert mlp() == WORKSPACE
    a = L.rmm_mlp_workspace_bytes(300, 512, 1024, 512, 0.5, 0.5)
    # the down projection's workspace plus X[:, I], the kept gate and up rows and the selection
    assert a >= L.rmm_linear_workspace_bytes(300, 1024, 512, 0.5) + 300 * 256 * 2 + 2 * 256 * 1024 * 2
    assert L.rmm_mlp_workspace_bytes(300, 512, 1024, 512, 1.0, 1.0) == 0


def test_int8_argument_errors(L):
    def li8(A=P16, n=4, d=512, lda=512, W=P16, m=1024, ldw=1024, s=P16, Y=P16, ldy=1024, rho=0.5, ws=None, wsb=0):
        return L.rmm_linear_int8(A, n, d, lda, W, m, ldw, s, Y, ldy, rho, None, ws, wsb, None)
    assert li8(s=None) == INVALID
    assert li8(rho=0.0) == INVALID
    assert li8(n=33) == UNSUPPORTED
    assert li8(m=1020, ldw=1024, ldy=1024) == UNSUPPORTED  # m not a multiple of 8
    assert li8(ldw=1028) == UNSUPPORTED                    # ldw not a multiple of 8
    assert li8() == WORKSPACE
    assert L.rmm_linear_int8_workspace_bytes(1, 8192, 28672, 1.0) > 0  # fp32 partial sums


def test_attention_argument_errors(L):
    def att(Q=P16, K=P16, V=P16, O=P16, b=1, hq=4, hkv=2, nq=256, nk=256, dh=128, causal=1, scale=0.1, rho=0.5,
            ws=None, wsb=0):
        return L.rmm_attention(Q, K, V, O, b, hq, hkv, nq, nk, dh, causal, scale, rho, None, ws, wsb, None)
    assert att(hkv=3) == INVALID
    assert att(V=None) == INVALID
    assert att(causal=2) == INVALID
    assert att(dh=64) == UNSUPPORTED
    assert att(nq=300, nk=256) == UNSUPPORTED   # causal with nq > nk
    assert att() == WORKSPACE
    assert L.rmm_attention_workspace_bytes(1, 4, 2, 256, 256, 128, 1.0) == 0
    # Q with the dropped dims zeroed, per query head
    assert L.rmm_attention_workspace_bytes(1, 4, 2, 256, 512, 128, 0.5) >= 4 * 256 * 128 * 2


@pytest.mark.parametrize("n", [1, 2])
@pytest.mark.parametrize("rho", [1.0, 0.9, 0.5, 0.01])
def test_int8_plan_fills_at_most_one_wave(L, n, rho):
    """The CUDA-core int8 GEMV (one or two activation rows) splits the kept rows into
    chunks, read back from the workspace size (scores, index set and chunks x n x m
    fp32 partial sums): the grid of 2048-column blocks x chunks fits in one wave of
    co-resident CTAs (4 or 3 per SM by the row count; 148 SMs when no device is
    visible) while every chunk holds at most 512 kept rows and a multiple of 16."""
    d, m = 8192, 28672
    k = L.rmm_k(rho, d)
    ws = L.rmm_linear_int8_workspace_bytes(n, d, m, rho)
    head = 0 if k == d else (d * 8 + 256 - 1) // 256 * 256 + (k * 4 + 256 - 1) // 256 * 256
    partial = ws - head
    assert partial > 0 and partial % (n * m * 4) == 0, (ws, head)
    chunks = partial // (n * m * 4)
    slots = {1: 4, 2: 3}.get(n, 2) * 148
    assert chunks * ((m + 2047) // 2048) <= slots
    chunk = -(-k // chunks)
    assert chunk <= 512
    # the chunk length the plan picks is a multiple of 16 covering k in `chunks` pieces
    lens = [ln for ln in range(16, 513, 16) if -(-k // ln) == chunks]
    assert lens, (k, chunks)


@pytest.mark.parametrize("n", [3, 8, 32])
def test_int8_tensor_core_workspace(L, n):
    """From three activation rows on, int8 weights run on the tensor cores: the
    workspace holds the scores, the index set, x[:, I] and the fp32 partials of the
    bf16 decode product's split (the same size as rmm_linear's decode workspace)."""
    d, m = 8192, 28672
    for rho in (0.5, 1.0):
        assert L.rmm_linear_int8_workspace_bytes(n, d, m, rho) == L.rmm_linear_workspace_bytes(n, d, m, rho)
