"""B200-native Reduced Matrix Multiplication (RMM).

Thin ctypes binding over the C ABI of ``librmm.so`` (declared in
``include/rmm.h``).  This module only marshals arguments -- every step of the
path (column scores, TopK selection, pack, tensor-core product) runs in the
library's sm_100a CUDA kernels.  PyTorch provides device memory and streams.

Importing this package does not load the library; the first call does, and
raises if ``librmm.so`` has not been built (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["lib", "rmm_k", "select", "linear", "gather_columns", "gather_rows", "gemm_packed", "gemm_gathered", "qk", "pv",
           "RMMError", "device_error", "library_path"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def library_path() -> str:
    return os.path.join(_HERE, "librmm.so")


class RMMError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p
_c_dbl = ctypes.c_double
_c_int = ctypes.c_int
_c_size = ctypes.c_size_t
_c_float = ctypes.c_float

_SIGNATURES = {
    "rmm_k": (_c_i64, [_c_dbl, _c_i64]),
    "rmm_select_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64]),
    "rmm_select": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_dbl, _c_p, _c_p, _c_p, _c_p,
                            _c_size, _c_p]),
    "rmm_linear_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_linear": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_dbl, _c_p, _c_p,
                            _c_size, _c_p]),
    "rmm_gather_columns": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_i64, _c_p]),
    "rmm_gather_rows": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_p, _c_i64, _c_p]),
    "rmm_gemm_packed": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_p]),
    "rmm_gemm_gathered": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_i64,
                                   _c_p]),
    "rmm_qk_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_qk": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_float, _c_dbl,
                        _c_p, _c_p, _c_size, _c_p]),
    "rmm_pv_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_pv": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_dbl, _c_p, _c_p,
                        _c_size, _c_p]),
    "rmm_attention_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_attention": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_int,
                               ctypes.c_float, _c_dbl, _c_p, _c_p, _c_size, _c_p]),
    "rmm_linear_int8_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_linear_int8": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_dbl,
                                 _c_p, _c_p, _c_size, _c_p]),
    "rmm_mlp_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_dbl, _c_dbl]),
    "rmm_mlp": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_p, _c_i64,
                         _c_p, _c_i64, _c_dbl, _c_dbl, _c_p, _c_p, _c_p, _c_size, _c_p]),
    "rmm_decode_qk_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_decode_qk": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64,
                               ctypes.c_float, _c_dbl, _c_p, _c_p, _c_size, _c_p]),
    "rmm_decode_pv_workspace_bytes": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_dbl]),
    "rmm_decode_pv": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_dbl,
                               _c_p, _c_p, _c_size, _c_p]),
    "rmm_status_string": (ctypes.c_char_p, [_c_int]),
    "rmm_last_error": (ctypes.c_char_p, []),
    "rmm_device_error": (_c_int, [ctypes.POINTER(ctypes.c_int32)]),
    "rmm_version": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """Load librmm.so (once) and declare the C signatures."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built; run `python -m input_adaptive_reduced_colnorm_b200.build`")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(status: int) -> None:
    if status != 0:
        L = lib()
        raise RMMError(status, f"{L.rmm_status_string(status).decode()}: {L.rmm_last_error().decode()}")


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require(t, name, dtype, dim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")


def _workspace(nbytes: int, device, workspace=None):
    import torch
    if nbytes == 0:
        return None
    if workspace is not None and workspace.numel() * workspace.element_size() >= nbytes:
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def rmm_k(rho: float, d: int) -> int:
    """k = ceil(rho * d) as the library computes it (-1 for invalid arguments)."""
    return int(lib().rmm_k(float(rho), int(d)))


def select(A, rho: float, *, causal: bool = False, colsq: bool = True, retained: bool = True, workspace=None):
    """Column scores and TopK index set of A ([n, d] or [batch, n, d], bf16, CUDA).

    Returns (idx int32 [batch?, k], colsq float64 [batch?, d] or None, retained float64 [batch?] or None)."""
    import torch
    _require(A, "A", torch.bfloat16)
    squeeze = A.dim() == 2
    A3 = A.unsqueeze(0) if squeeze else A
    if A3.dim() != 3 or A3.stride(2) != 1:
        raise ValueError("A must be [n, d] or [batch, n, d] with unit column stride")
    batch, n, d = A3.shape
    lda = A3.stride(1)
    bstride = A3.stride(0) if batch > 1 else n * lda
    k = rmm_k(rho, d)
    if k < 0:
        raise RMMError(1, f"invalid rho {rho}")
    dev = A.device
    idx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    cs = torch.empty((batch, d), dtype=torch.float64, device=dev) if colsq else None
    rt = torch.empty((batch,), dtype=torch.float64, device=dev) if retained else None
    L = lib()
    ws = None if colsq else _workspace(L.rmm_select_workspace_bytes(batch, n, d), dev, workspace)
    _check(L.rmm_select(_ptr(A3), batch, bstride, n, d, lda, int(causal), float(rho), _ptr(idx), _ptr(cs), _ptr(rt),
                        _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    if squeeze:
        idx = idx[0]
        cs = None if cs is None else cs[0]
        rt = None if rt is None else rt[0]
    return idx, cs, rt


def linear(A, B, rho: float, *, out=None, return_idx: bool = False, workspace=None):
    """Y = A[:, I] . B[I, :] with I the TopK column-norm set of A.

    A [n, d] bf16 (row stride may exceed d), B [d, m] bf16 (contraction index on
    rows), both CUDA.  Returns Y [n, m] bf16 (and idx int32 [k] if asked)."""
    import torch
    _require(A, "A", torch.bfloat16, 2)
    _require(B, "B", torch.bfloat16, 2)
    if A.stride(1) != 1 or B.stride(1) != 1:
        raise ValueError("A and B need unit column stride")
    n, d = A.shape
    d2, m = B.shape
    if d2 != d:
        raise ValueError(f"contraction mismatch: A has {d} columns, B has {d2} rows")
    dev = A.device
    if out is None:
        out = torch.empty((n, m), dtype=torch.bfloat16, device=dev)
    _require(out, "out", torch.bfloat16, 2)
    k = rmm_k(rho, d)
    idx = torch.empty((max(k, 0),), dtype=torch.int32, device=dev) if return_idx else None
    L = lib()
    ws = _workspace(L.rmm_linear_workspace_bytes(n, d, m, float(rho)), dev, workspace)
    _check(L.rmm_linear(_ptr(A), n, d, A.stride(0), _ptr(B), m, B.stride(0), _ptr(out), out.stride(0), float(rho),
                        _ptr(idx), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def gather_columns(A, idx, out=None, ld_pack=None):
    """A_pack[:, :k] = A[:, idx], zero-padded; returns the [n, ld_pack] buffer."""
    import torch
    _require(A, "A", torch.bfloat16, 2)
    n, d = A.shape
    k = idx.numel()
    if out is None:
        ld = ((k + 7) // 8) * 8 if ld_pack is None else ld_pack
        out = torch.empty((n, ld), dtype=torch.bfloat16, device=A.device)
    _check(lib().rmm_gather_columns(_ptr(A), n, d, A.stride(0), _ptr(idx), k, _ptr(out), out.stride(0),
                                    _stream(A.device)))
    return out


def gather_rows(B, idx, out=None, ld_pack=None):
    """B_pack[t, :] = B[idx[t], :]; returns the [k, ld_pack] buffer."""
    import torch
    _require(B, "B", torch.bfloat16, 2)
    d, m = B.shape
    k = idx.numel()
    if out is None:
        ld = ((m + 7) // 8) * 8 if ld_pack is None else ld_pack
        out = torch.empty((k, ld), dtype=torch.bfloat16, device=B.device)
    _check(lib().rmm_gather_rows(_ptr(B), d, m, B.stride(0), _ptr(idx), k, _ptr(out), out.stride(0),
                                 _stream(B.device)))
    return out


def gemm_packed(A_pack, k, B_pack, m, out=None):
    """Y = A_pack[:, :k] . B_pack[:k, :m] on the tensor cores."""
    import torch
    _require(A_pack, "A_pack", torch.bfloat16, 2)
    _require(B_pack, "B_pack", torch.bfloat16, 2)
    n = A_pack.shape[0]
    if out is None:
        out = torch.empty((n, m), dtype=torch.bfloat16, device=A_pack.device)
    _check(lib().rmm_gemm_packed(_ptr(A_pack), n, int(k), A_pack.stride(0), _ptr(B_pack), int(m), B_pack.stride(0),
                                 _ptr(out), out.stride(0), _stream(A_pack.device)))
    return out


def gemm_gathered(A_pack, k, B, idx, out=None):
    """Y = A_pack[:, :k] . B[idx[:k], :] with the kept rows of B read through the index set."""
    import torch
    _require(A_pack, "A_pack", torch.bfloat16, 2)
    _require(B, "B", torch.bfloat16, 2)
    _require(idx, "idx", torch.int32, 1)
    n = A_pack.shape[0]
    d, m = B.shape
    if out is None:
        out = torch.empty((n, m), dtype=torch.bfloat16, device=A_pack.device)
    _check(lib().rmm_gemm_gathered(_ptr(A_pack), n, int(k), A_pack.stride(0), _ptr(B), d, m, B.stride(0), _ptr(idx),
                                   _ptr(out), out.stride(0), _stream(A_pack.device)))
    return out


def qk(Q, K, rho: float, *, causal: bool = True, scale: float = 1.0, out=None, return_idx: bool = False,
       workspace=None):
    """Reduced attention scores.  Q [B, Hq, nq, dh], K [B, Hkv, nk, dh] bf16 contiguous
    -> S [B, Hq, nq, nk] float32 (-inf where causally masked)."""
    import torch
    _require(Q, "Q", torch.bfloat16, 4)
    _require(K, "K", torch.bfloat16, 4)
    if not (Q.is_contiguous() and K.is_contiguous()):
        raise ValueError("Q and K must be contiguous")
    b, hq, nq, dh = Q.shape
    b2, hkv, nk, dh2 = K.shape
    if b2 != b or dh2 != dh:
        raise ValueError("Q / K shape mismatch")
    dev = Q.device
    if out is None:
        out = torch.empty((b, hq, nq, nk), dtype=torch.float32, device=dev)
    k = rmm_k(rho, dh)
    idx = torch.empty((b, hq, max(k, 0)), dtype=torch.int32, device=dev) if return_idx else None
    L = lib()
    ws = _workspace(L.rmm_qk_workspace_bytes(b, hq, hkv, nq, nk, dh, float(rho)), dev, workspace)
    _check(L.rmm_qk(_ptr(Q), _ptr(K), _ptr(out), b, hq, hkv, nq, nk, dh, int(causal), float(scale), float(rho),
                    _ptr(idx), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def pv(P, V, rho: float, *, causal: bool = True, out=None, return_idx: bool = False, workspace=None):
    """Reduced attention output.  P [B, H, nq, nk], V [B, Hkv, nk, dh] bf16 contiguous
    -> O [B, H, nq, dh] bf16."""
    import torch
    _require(P, "P", torch.bfloat16, 4)
    _require(V, "V", torch.bfloat16, 4)
    if not (P.is_contiguous() and V.is_contiguous()):
        raise ValueError("P and V must be contiguous")
    b, h, nq, nk = P.shape
    b2, hkv, nk2, dh = V.shape
    if b2 != b or nk2 != nk:
        raise ValueError("P / V shape mismatch")
    dev = P.device
    if out is None:
        out = torch.empty((b, h, nq, dh), dtype=torch.bfloat16, device=dev)
    k = rmm_k(rho, nk)
    idx = torch.empty((b, h, max(k, 0)), dtype=torch.int32, device=dev) if return_idx else None
    L = lib()
    ws = _workspace(L.rmm_pv_workspace_bytes(b, h, hkv, nq, nk, dh, float(rho)), dev, workspace)
    _check(L.rmm_pv(_ptr(P), _ptr(V), _ptr(out), b, h, hkv, nq, nk, dh, int(causal), float(rho), _ptr(idx),
                    _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def attention(Q, K, V, rho: float, *, causal: bool = True, scale: float = 1.0, out=None, return_idx: bool = False,
              workspace=None):
    """Fused attention with a reduced score product: O = softmax(scale Q_I K_I^T) V per
    query head.  Q [B, Hq, nq, 128], K / V [B, Hkv, nk, 128] bf16 contiguous -> O
    [B, Hq, nq, 128] bf16."""
    import torch
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V")):
        _require(t, nm, torch.bfloat16, 4)
        if not t.is_contiguous():
            raise ValueError(f"{nm} must be contiguous")
    b, hq, nq, dh = Q.shape
    b2, hkv, nk, dh2 = K.shape
    if b2 != b or dh2 != dh or V.shape != K.shape:
        raise ValueError("Q / K / V shape mismatch")
    dev = Q.device
    if out is None:
        out = torch.empty((b, hq, nq, dh), dtype=torch.bfloat16, device=dev)
    k = rmm_k(rho, dh)
    idx = torch.empty((b, hq, max(k, 0)), dtype=torch.int32, device=dev) if return_idx else None
    Lb = lib()
    ws = _workspace(Lb.rmm_attention_workspace_bytes(b, hq, hkv, nq, nk, dh, float(rho)), dev, workspace)
    _check(Lb.rmm_attention(_ptr(Q), _ptr(K), _ptr(V), _ptr(out), b, hq, hkv, nq, nk, dh, int(causal), float(scale),
                            float(rho), _ptr(idx), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def linear_int8(A, Wq, scale, rho: float, *, out=None, return_idx: bool = False, workspace=None):
    """Y = (A[:, I] Wq[I, :]) * scale with I chosen on A (decode, n <= 32 rows).
    A [n, d] bf16, Wq [d, m] int8, scale [m] float32, all CUDA."""
    import torch
    _require(A, "A", torch.bfloat16, 2)
    _require(Wq, "Wq", torch.int8, 2)
    _require(scale, "scale", torch.float32, 1)
    n, d = A.shape
    d2, m = Wq.shape
    if d2 != d or scale.numel() != m:
        raise ValueError("A / Wq / scale shape mismatch")
    dev = A.device
    if out is None:
        out = torch.empty((n, m), dtype=torch.bfloat16, device=dev)
    Lb = lib()
    idx = torch.empty((max(rmm_k(rho, d), 0),), dtype=torch.int32, device=dev) if return_idx else None
    ws = _workspace(Lb.rmm_linear_int8_workspace_bytes(n, d, m, float(rho)), dev, workspace)
    _check(Lb.rmm_linear_int8(_ptr(A), n, d, A.stride(0), _ptr(Wq), m, Wq.stride(0), _ptr(scale), _ptr(out),
                              out.stride(0), float(rho), _ptr(idx), _ptr(ws), 0 if ws is None else ws.numel(),
                              _stream(dev)))
    return (out, idx) if return_idx else out


def mlp(X, Wg, Wu, Wd, rho_gu: float, rho_down: float, *, H=None, out=None, return_idx: bool = False,
        workspace=None):
    """Gated MLP block: H = SiLU(X_I Wg[I]) * (X_I Wu[I]) with one index set I on X for
    gate and up, then Y = RMM(H, Wd) with its own selection.  X [n, d], Wg / Wu [d, f],
    Wd [f, m] bf16 CUDA.  Returns Y (and H, idx_gu, idx_down if asked)."""
    import torch
    for t, nm in ((X, "X"), (Wg, "Wg"), (Wu, "Wu"), (Wd, "Wd")):
        _require(t, nm, torch.bfloat16, 2)
    n, d = X.shape
    d2, f = Wg.shape
    if Wu.shape != Wg.shape or d2 != d or Wd.shape[0] != f:
        raise ValueError("MLP shape mismatch")
    if Wg.stride(0) != Wu.stride(0):
        raise ValueError("Wg and Wu must share a row stride")
    m = Wd.shape[1]
    dev = X.device
    if H is None:
        H = torch.empty((n, f), dtype=torch.bfloat16, device=dev)
    if out is None:
        out = torch.empty((n, m), dtype=torch.bfloat16, device=dev)
    Lb = lib()
    i1 = torch.empty((max(rmm_k(rho_gu, d), 0),), dtype=torch.int32, device=dev) if return_idx else None
    i2 = torch.empty((max(rmm_k(rho_down, f), 0),), dtype=torch.int32, device=dev) if return_idx else None
    ws = _workspace(Lb.rmm_mlp_workspace_bytes(n, d, f, m, float(rho_gu), float(rho_down)), dev, workspace)
    _check(Lb.rmm_mlp(_ptr(X), n, d, X.stride(0), _ptr(Wg), _ptr(Wu), f, Wg.stride(0), _ptr(Wd), m, Wd.stride(0),
                      _ptr(H), H.stride(0), _ptr(out), out.stride(0), float(rho_gu), float(rho_down), _ptr(i1),
                      _ptr(i2), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, H, i1, i2) if return_idx else out


def decode_qk(Q, Kt, rho: float, *, nk=None, scale: float = 1.0, out=None, return_idx: bool = False,
              workspace=None):
    """Decode scores against a dim-major key cache.  Q [B, Hq, dh], Kt [B, Hkv, dh, L]
    (tokens along the last axis, the first nk valid; L a multiple of 8) -> S [B, Hq, nk]
    fp32.  One index set per key/value group, chosen on the group's query rows."""
    import torch
    _require(Q, "Q", torch.bfloat16, 3)
    _require(Kt, "Kt", torch.bfloat16, 4)
    if not (Q.is_contiguous() and Kt.is_contiguous()):
        raise ValueError("Q and Kt must be contiguous")
    b, hq, dh = Q.shape
    b2, hkv, dh2, L = Kt.shape
    if b2 != b or dh2 != dh:
        raise ValueError("Q / Kt shape mismatch")
    nk = L if nk is None else int(nk)
    dev = Q.device
    if out is None:
        out = torch.empty((b, hq, (nk + 3) // 4 * 4), dtype=torch.float32, device=dev)[:, :, :nk]
    k = rmm_k(rho, dh)
    idx = torch.empty((b, hkv, max(k, 0)), dtype=torch.int32, device=dev) if return_idx else None
    Lb = lib()
    ws = _workspace(Lb.rmm_decode_qk_workspace_bytes(b, hq, hkv, dh, float(rho)), dev, workspace)
    _check(Lb.rmm_decode_qk(_ptr(Q), _ptr(Kt), _ptr(out), b, hq, hkv, dh, nk, L, out.stride(1), float(scale),
                            float(rho), _ptr(idx), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def decode_pv(P, V, rho: float, *, nk=None, out=None, return_idx: bool = False, workspace=None):
    """Decode attention output against a token-major value cache.  P [B, Hq, L]
    (probabilities of the one query row, the first nk valid; L a multiple of 8),
    V [B, Hkv, cap, dh] -> O [B, Hq, dh] bf16.  One index set per key/value group."""
    import torch
    _require(P, "P", torch.bfloat16, 3)
    _require(V, "V", torch.bfloat16, 4)
    if not (P.is_contiguous() and V.is_contiguous()):
        raise ValueError("P and V must be contiguous")
    b, hq, L = P.shape
    b2, hkv, cap, dh = V.shape
    if b2 != b:
        raise ValueError("P / V shape mismatch")
    nk = min(L, cap) if nk is None else int(nk)
    dev = P.device
    if out is None:
        out = torch.empty((b, hq, dh), dtype=torch.bfloat16, device=dev)
    k = rmm_k(rho, nk)
    idx = torch.empty((b, hkv, max(k, 0)), dtype=torch.int32, device=dev) if return_idx else None
    Lb = lib()
    ws = _workspace(Lb.rmm_decode_pv_workspace_bytes(b, hq, hkv, nk, dh, float(rho)), dev, workspace)
    _check(Lb.rmm_decode_pv(_ptr(P), _ptr(V), _ptr(out), b, hq, hkv, nk, L, cap, dh, float(rho), _ptr(idx),
                            _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev)))
    return (out, idx) if return_idx else out


def device_error() -> int:
    """Read and clear the device-side error word (synchronises the device)."""
    v = ctypes.c_int32(0)
    _check(lib().rmm_device_error(ctypes.byref(v)))
    return int(v.value)
