"""CPU oracle for Reduced Matrix Multiplication (RMM) -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, the package's smoke check and the benchmark's CPU-baseline
leg may import or run this module.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

It restates, plainly and slowly in float64 with numpy, what RMM computes.  Every
function cites the page passage it follows.  Pages (by title):

  [DD]   "Algorithm Deep-Dive: RMM -- TopK Column-Norm Slicing: Formulas, 1B-70B
          Results, and the Attention/MLP Asymmetry" (hackcv.com)
  [KB]   "RMM：把 Transformer 矩阵乘法切到刚好够用" (kaelemshawn.blog)
  [GS]   "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction
          for LLM Inference", Technical Summary (gist.science)

Readings where the pages are silent (each is also pinned by a test):
  * k = ceil(rho*d), computed as ceil(x - 1e-9*x) with x = rho*d so that a
    product such as 0.1*30 = 3.0000000000000004 still gives 3; clamped to [1, d].
  * Ties in the column norm: the lower index wins.  The index set is returned
    in ascending order.
  * Retained energy = sum_{j in I} s_j^2 / sum_j s_j^2.
  * Causal attention (QK^T and PV) is bottom-right aligned: key j is visible to
    query i iff j <= i + (nk - nq).  Masked scores are -inf; masked entries of
    P are treated as zero (they are neither read for the norms nor multiplied).
  * GQA: query head h reads key/value head h // (Hq // Hkv).
  * Decode attention (one query row per head, keys and values in a cache): the
    G = Hq / Hkv query rows that share a key/value head are the rows of A, so
    each key/value head gets ONE index set, chosen on the column norms of its
    group's rows, and its cache is read once for the whole group.  (Per-head
    sets would make the G heads of a group read G different subsets of the same
    cache.)  For Hq = Hkv this is per head.

Parity: every function here is pinned by tests/test_oracle.py against
hand-derived fixtures, closed forms, brute force or invariants; none is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "retention_count", "column_sq_norms", "column_norms", "topk_ascending",
    "retained_energy", "select", "reduced_product", "error_bound", "rmm_linear",
    "rmm_linear_rows", "kv_head", "rmm_qk", "rmm_qk_rows", "rmm_pv", "rmm_pv_rows",
    "near_tie_band", "rmm_decode_qk", "rmm_decode_pv", "silu", "rmm_mlp_gate_up", "rmm_mlp",
    "rmm_linear_int8", "rmm_attention", "qk_scores_rows", "pv_output_rows", "attention_rows",
    "int8_product_rows", "mlp_gate_up_rows", "rmm_attention_rows",
]


def retention_count(rho: float, d: int) -> int:
    """k = ceil(rho * d), the number of contraction indices kept.

    [DD] "The retention-ratio (rho) Knob": rho in (0, 1] keeps ceil(rho d) dims;
    [KB] "先把...想清楚": |I| = ceil(rho d); [GS] Methodology, Selection Strategy.
    """
    rho = float(rho)
    d = int(d)
    if not (rho > 0.0 and rho <= 1.0) or d < 1:
        raise ValueError(f"rho must lie in (0, 1] and d >= 1 (rho={rho}, d={d})")
    x = rho * d
    k = math.ceil(x - 1e-9 * x)
    return max(1, min(d, k))


def _visible_cols(i: int, nq: int, nk: int) -> int:
    """Number of key positions visible to query row i under bottom-right causal alignment."""
    return max(0, min(nk, i + (nk - nq) + 1))


def column_sq_norms(A: np.ndarray, causal: bool = False) -> np.ndarray:
    """q_j = sum_i A[i, j]^2 in float64, summed in row order.

    The importance score is the activation column L2 norm s_j = ||A[:, j]||_2
    ([DD] "Contraction-Dimension TopK Selection"; [GS] Selection Strategy); this
    returns its square.  With ``causal`` the entries above the bottom-right
    aligned diagonal are treated as zero (attention probabilities P).
    """
    A = np.asarray(A, dtype=np.float64)
    n, d = A.shape
    q = np.zeros(d, dtype=np.float64)
    for i in range(n):
        lim = _visible_cols(i, n, d) if causal else d
        if lim > 0:
            row = A[i, :lim]
            q[:lim] += row * row
    return q


def column_norms(A: np.ndarray, causal: bool = False) -> np.ndarray:
    """s_j = ||A[:, j]||_2 ([DD] "Contraction-Dimension TopK Selection")."""
    return np.sqrt(column_sq_norms(A, causal))


def topk_ascending(s: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, ties to the lower index, returned ascending.

    [DD] "take TopK-largest ceil(rho d)"; [GS] "The top-k indices with the
    highest scores are retained".  Order: by score descending, then index
    ascending; keep the first k; sort the kept indices ascending.
    """
    s = np.asarray(s, dtype=np.float64)
    d = s.shape[0]
    if not (1 <= k <= d):
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(d), -s))
    return np.sort(order[:k]).astype(np.int64)


def retained_energy(q: np.ndarray, I: np.ndarray) -> float:
    """sum_{j in I} s_j^2 / sum_j s_j^2 (reading of the pages' "retained activation
    energy", [DD] "Attention vs MLP: structural asymmetry", supplementary note)."""
    total = float(np.sum(q))
    return float(np.sum(q[I])) / total if total > 0 else 1.0


def near_tie_band(s: np.ndarray, k: int, rel: float = 1e-5) -> np.ndarray:
    """Indices j whose norm lies within ``rel`` (relative) of the k-th largest norm.

    Selections that differ only inside this band are all correct up to rounding
    of the scores; parity tests accept (and log) differences there."""
    s = np.asarray(s, dtype=np.float64)
    kth = np.sort(s)[::-1][k - 1]
    return np.nonzero(np.abs(s - kth) <= rel * abs(kth))[0]


def select(A: np.ndarray, rho: float, causal: bool = False):
    """Score, count and TopK: returns (I, q, retained) for one activation matrix.

    [DD] "Core Approach (Formula Level)"; [GS] Methodology items 1-2.
    """
    A = np.asarray(A, dtype=np.float64)
    d = A.shape[1]
    k = retention_count(rho, d)
    q = column_sq_norms(A, causal)
    I = topk_ascending(np.sqrt(q), k)
    return I, q, retained_energy(q, I)


def reduced_product(A: np.ndarray, B: np.ndarray, I: np.ndarray) -> np.ndarray:
    """RMM_rho(A, B) = A[:, I] . B[I, :] in float64.

    [DD] "Contraction-Dimension TopK Selection"; [KB] "RMMρ(A, B) = A[:, I] B[I, :]";
    [GS] Core Mechanism.  Weights are not modified; rows of B outside I are skipped.
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return A[:, I] @ B[I, :]


def error_bound(A: np.ndarray, B: np.ndarray, I: np.ndarray) -> float:
    """sum_{j not in I} ||A[:, j]||_2 * ||B[j, :]||_2 ([DD] "Properties", error bound)."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    keep = np.zeros(A.shape[1], dtype=bool)
    keep[I] = True
    s = column_norms(A)
    b = np.sqrt(np.sum(B * B, axis=1))
    return float(np.sum(s[~keep] * b[~keep]))


def rmm_linear(A: np.ndarray, B: np.ndarray, rho: float):
    """Reduced linear projection Y = X[:, I] W[I, :] with I chosen on X.

    [DD] "Component mapping": MLP/linear projections select along the activation
    hidden dim; [KB] "在线性投影和 MLP 里"; [GS] Application Scope (XW).
    Returns dict(Y, I, q, retained).
    """
    I, q, ret = select(A, rho)
    return {"Y": reduced_product(A, B, I), "I": I, "q": q, "retained": ret}


def rmm_linear_rows(A: np.ndarray, B: np.ndarray, I: np.ndarray, rows) -> np.ndarray:
    """Rows ``rows`` of A[:, I] . B[I, :] (for sampled checks of large products)."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    rows = np.asarray(rows)
    return A[rows][:, I] @ B[I, :]


def kv_head(h: int, hq: int, hkv: int) -> int:
    """Key/value head read by query head h under GQA: h // (Hq // Hkv)."""
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (hq // hkv)


def _check_index_set(I, d, what):
    I = np.asarray(I, dtype=np.int64).reshape(-1)
    if I.size < 1 or I.size > d or np.any(I < 0) or np.any(I >= d) or np.any(np.diff(I) <= 0):
        raise ValueError(f"{what}: the index set must be strictly ascending within [0, {d})")
    return I


def qk_scores_rows(Qh: np.ndarray, Kg: np.ndarray, I, rows=None, causal: bool = True, scale: float = 1.0):
    """Rows ``rows`` of one head's reduced scores on a GIVEN index set I:
        S[i, j] = scale * sum_{t in I} Qh[i, t] * Kg[j, t],
    -inf where key j is not visible to query i (bottom-right causal alignment).

    [DD] "Component mapping": QK^T contracts over the kept head-feature dims only;
    under GQA the key head gathers the query head's dims.  Qh [nq, dh], Kg [nk, dh].
    The product on the index set the library chose is what a parity check compares
    when two sets differ only inside the near-tie band."""
    Qh = np.asarray(Qh, dtype=np.float64)
    Kg = np.asarray(Kg, dtype=np.float64)
    nq, dh = Qh.shape
    nk = Kg.shape[0]
    I = _check_index_set(I, dh, "qk_scores_rows")
    r = np.arange(nq) if rows is None else np.asarray(rows)
    S = scale * (Qh[r][:, I] @ Kg[:, I].T)
    if causal:
        vis = np.array([_visible_cols(i, nq, nk) for i in r])
        S[np.arange(nk)[None, :] >= vis[:, None]] = -np.inf
    return S


def _qk_head(Qh, Kg, rho, causal, scale, rows=None, I=None):
    nq, dh = Qh.shape
    if I is None:
        k = retention_count(rho, dh)
        q = column_sq_norms(Qh)
        I = topk_ascending(np.sqrt(q), k)
    I = _check_index_set(I, dh, "qk")
    return qk_scores_rows(Qh, Kg, I, rows, causal, scale), I


def rmm_qk(Q: np.ndarray, K: np.ndarray, rho: float, causal: bool = True, scale: float = 1.0):
    """Reduced attention scores S_h = scale * Q_h[:, I_h] K_g(h)[:, I_h]^T per query head.

    [DD] "Component mapping": QK^T selects along the head feature dim with score =
    Q column norm; under GQA the selection is made on Q per head and K gathers the
    corresponding dims.  [KB] "计算 attention score 时"; [GS] Application Scope.
    Q [B, Hq, nq, dh], K [B, Hkv, nk, dh] -> S [B, Hq, nq, nk] (float64, -inf where
    masked), I [B, Hq, k].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    Bsz, hq, nq, dh = Q.shape
    hkv, nk = K.shape[1], K.shape[2]
    k = retention_count(rho, dh)
    S = np.empty((Bsz, hq, nq, nk))
    I = np.empty((Bsz, hq, k), dtype=np.int64)
    for b in range(Bsz):
        for h in range(hq):
            S[b, h], I[b, h] = _qk_head(Q[b, h], K[b, kv_head(h, hq, hkv)], rho, causal, scale)
    return {"S": S, "I": I}


def rmm_qk_rows(Qh: np.ndarray, Kg: np.ndarray, rho: float, rows, causal=True, scale=1.0, I=None):
    """Rows ``rows`` of one head's reduced scores: Qh [nq, dh] (the query head),
    Kg [nk, dh] (its GQA key head).  I = the oracle's own TopK of Qh's column norms,
    or the given index set.  Returns (S_rows, I)."""
    return _qk_head(np.asarray(Qh, dtype=np.float64), np.asarray(Kg, dtype=np.float64),
                    rho, causal, scale, rows, I)


def pv_output_rows(Ph: np.ndarray, Vg: np.ndarray, I, rows=None, causal: bool = True):
    """Rows ``rows`` of one head's reduced attention output on a GIVEN index set I:
        O[i, :] = sum_{j in I, j visible to i} Ph[i, j] * Vg[j, :]
    (entries of P above the bottom-right aligned diagonal count as zero).

    [DD] "Component mapping": PV contracts over the kept token positions only, the
    V rows of those positions gathered.  Ph [nq, nk], Vg [nk, dh]."""
    Ph = np.asarray(Ph, dtype=np.float64)
    Vg = np.asarray(Vg, dtype=np.float64)
    nq, nk = Ph.shape
    I = _check_index_set(I, nk, "pv_output_rows")
    r = np.arange(nq) if rows is None else np.asarray(rows)
    Pr = Ph[r][:, I].copy()
    if causal:
        vis = np.array([_visible_cols(i, nq, nk) for i in r])
        Pr[I[None, :] >= vis[:, None]] = 0.0
    return Pr @ Vg[I, :]


def _pv_head(Ph, Vg, rho, causal, rows=None, I=None):
    nq, nk = Ph.shape
    q = column_sq_norms(Ph, causal)
    if I is None:
        k = retention_count(rho, nk)
        I = topk_ascending(np.sqrt(q), k)
    I = _check_index_set(I, nk, "pv")
    return pv_output_rows(Ph, Vg, I, rows, causal), I, q


def rmm_pv(P: np.ndarray, V: np.ndarray, rho: float, causal: bool = True):
    """Reduced attention output O_h = P_h[:, I_h] V_g(h)[I_h, :] per head.

    [DD] "Component mapping": PV optionally selects along token positions;
    [KB] "计算 attention output 时": P's norm over positions decides which V rows
    take part; [GS] Application Scope.  The score of key position j is the norm of
    column j of P over all query rows.  P [B, H, nq, nk], V [B, Hkv, nk, dh] ->
    O [B, H, nq, dh], I [B, H, k].
    """
    P = np.asarray(P, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Bsz, h_, nq, nk = P.shape
    hkv, dh = V.shape[1], V.shape[3]
    k = retention_count(rho, nk)
    O = np.empty((Bsz, h_, nq, dh))
    I = np.empty((Bsz, h_, k), dtype=np.int64)
    for b in range(Bsz):
        for h in range(h_):
            O[b, h], I[b, h], _ = _pv_head(P[b, h], V[b, kv_head(h, h_, hkv)], rho, causal)
    return {"O": O, "I": I}


def rmm_pv_rows(Ph: np.ndarray, Vg: np.ndarray, rho: float, rows, causal=True, I=None):
    """Rows ``rows`` of one head's reduced PV output, on the oracle's own TopK of the
    column norms of Ph or on the given index set.  Returns (O_rows, I, q)."""
    return _pv_head(np.asarray(Ph, dtype=np.float64), np.asarray(Vg, dtype=np.float64), rho, causal, rows, I)


def _group(hq: int, hkv: int) -> int:
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // hkv


def rmm_decode_qk(Q: np.ndarray, Kt: np.ndarray, rho: float, scale: float = 1.0, nk=None):
    """Decode scores against a key cache: per key/value group g of batch item b,
    A = Q[b, g G:(g+1) G, :] (the group's G query rows, [G, dh]), I_g = TopK of the
    column norms of A over the head-feature dims, and
        S[b, h, j] = scale * sum_{t in I_g} Q[b, h, t] * Kt[b, g, t, j],   j < nk.

    [DD] "Component mapping" (QK^T selects along the head feature dim by the Q
    column norm; K gathers those dims) and "Engineering Notes" (decode prunes
    attention); [KB] "计算 attention score 时".  The key cache is dim-major
    (Kt [B, Hkv, dh, L], tokens along the last axis), so the kept dims are whole
    rows of it.  Q [B, Hq, dh] -> S [B, Hq, nk], I [B, Hkv, k].
    """
    Q = np.asarray(Q, dtype=np.float64)
    Kt = np.asarray(Kt, dtype=np.float64)
    Bsz, hq, dh = Q.shape
    hkv, L = Kt.shape[1], Kt.shape[3]
    nk = L if nk is None else int(nk)
    G = _group(hq, hkv)
    k = retention_count(rho, dh)
    S = np.empty((Bsz, hq, nk))
    I = np.empty((Bsz, hkv, k), dtype=np.int64)
    for b in range(Bsz):
        for g in range(hkv):
            A = Q[b, g * G:(g + 1) * G]
            Ig = topk_ascending(column_norms(A), k)
            S[b, g * G:(g + 1) * G] = scale * reduced_product(A, Kt[b, g][:, :nk], Ig)
            I[b, g] = Ig
    return {"S": S, "I": I}


def rmm_decode_pv(P: np.ndarray, V: np.ndarray, rho: float, nk=None):
    """Decode attention output against a value cache: per key/value group g of
    batch item b, A = P[b, g G:(g+1) G, :nk] (the group's G probability rows),
    I_g = TopK of the column norms of A over the token positions, and
        O[b, h, :] = sum_{j in I_g} P[b, h, j] * V[b, g, j, :].

    [DD] "Component mapping" (PV selects along token positions) and "Engineering
    Notes" (decode prunes attention); [KB] "计算 attention output 时": only the
    positions where P has the larger norm let their V rows take part.
    P [B, Hq, L] (first nk valid), V [B, Hkv, L, dh] -> O [B, Hq, dh], I [B, Hkv, k].
    """
    P = np.asarray(P, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Bsz, hq, L = P.shape
    hkv, dh = V.shape[1], V.shape[3]
    nk = L if nk is None else int(nk)
    G = _group(hq, hkv)
    k = retention_count(rho, nk)
    O = np.empty((Bsz, hq, dh))
    I = np.empty((Bsz, hkv, k), dtype=np.int64)
    for b in range(Bsz):
        for g in range(hkv):
            A = P[b, g * G:(g + 1) * G, :nk]
            Ig = topk_ascending(column_norms(A), k)
            O[b, g * G:(g + 1) * G] = reduced_product(A, V[b, g, :nk], Ig)
            I[b, g] = Ig
    return {"O": O, "I": I}


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x / (1 + exp(-x)) in float64 (the gate nonlinearity of the MLP block)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def rmm_mlp_gate_up(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, rho: float):
    """Gate and up projections of the MLP block with ONE index set I chosen on X
    (both contract the same input X), then H = SiLU(X_I Wg[I, :]) * (X_I Wu[I, :]).

    [DD] "Attention vs MLP: structural asymmetry" (MLP Up / Down / whole MLP reduced
    separately) and "Engineering Notes" (conservative MLP rho); [KB] the MLP Up / Gate /
    Down component analysis.  Returns dict(H, I, G, U).
    """
    I, _, _ = select(X, rho)
    H, G, U = mlp_gate_up_rows(X, Wg, Wu, I, rows=None, parts=True)
    return {"H": H, "I": I, "G": G, "U": U}


def mlp_gate_up_rows(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, I, rows=None, parts: bool = False):
    """Rows ``rows`` of H = SiLU(X[:, I] Wg[I, :]) * (X[:, I] Wu[I, :]) on a GIVEN index
    set I (the one set shared by gate and up, see ``rmm_mlp_gate_up``).  With ``parts``
    returns (H, G, U)."""
    X = np.asarray(X, dtype=np.float64)
    I = _check_index_set(I, X.shape[1], "mlp_gate_up_rows")
    r = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    Xr = X[r]
    G = reduced_product(Xr, Wg, I)
    U = reduced_product(Xr, Wu, I)
    H = silu(G) * U
    return (H, G, U) if parts else H


def rmm_mlp(X, Wg, Wu, Wd, rho_gu: float, rho_down: float):
    """The whole MLP block: H from ``rmm_mlp_gate_up`` (one selection on X), then the
    down projection Y = H[:, J] Wd[J, :] with its own rho and J chosen on H's column
    norms (the down input is SiLU(gate) * up).  Returns dict(H, I_gu, Y, I_down)."""
    gu = rmm_mlp_gate_up(X, Wg, Wu, rho_gu)
    down = rmm_linear(gu["H"], Wd, rho_down)
    return {"H": gu["H"], "I_gu": gu["I"], "Y": down["Y"], "I_down": down["I"]}


def rmm_linear_int8(A: np.ndarray, Wq: np.ndarray, scale: np.ndarray, rho: float):
    """Reduced projection with int8 weights: W = Wq * scale[None, :] (one scale per
    output column), I chosen on A as in ``rmm_linear``, and
        Y = (A[:, I] . Wq[I, :]) * scale[None, :].

    [GS] "Compatibility" (the method works with INT8 weight quantization) and [DD]
    "Compatibility & generalization" (INT8 + RMM: lower precision and fewer FLOPs
    stack): the selection and the kept rows are those of the bf16 case; only the
    stored weights are int8.  Returns dict(Y, I).
    """
    A = np.asarray(A, dtype=np.float64)
    I, _, _ = select(A, rho)
    return {"Y": int8_product_rows(A, Wq, scale, I), "I": I}


def int8_product_rows(A: np.ndarray, Wq: np.ndarray, scale: np.ndarray, I, rows=None) -> np.ndarray:
    """Rows ``rows`` of (A[:, I] . Wq[I, :]) * scale[None, :] on a GIVEN index set I
    (int8 codes widened exactly, one scale per output column; see ``rmm_linear_int8``)."""
    A = np.asarray(A, dtype=np.float64)
    Wq = np.asarray(Wq, dtype=np.float64)
    scale = np.asarray(scale, dtype=np.float64)
    I = _check_index_set(I, A.shape[1], "int8_product_rows")
    r = np.arange(A.shape[0]) if rows is None else np.asarray(rows)
    return (A[r][:, I] @ Wq[I, :]) * scale[None, :]


def rmm_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, rho: float, causal: bool = True,
                  scale: float = 1.0):
    """Attention whose score product is reduced: per query head h,
        S_h = scale * Q_h[:, I_h] K_g(h)[:, I_h]^T   (I_h = TopK of Q_h's column norms,
                                                    -inf above the causal diagonal)
        O_h = softmax_rows(S_h) V_g(h)               (the value product is not reduced)

    [DD] "Component mapping" (QK^T selects head dims on Q) and "Attention vs MLP"
    (Table 16: attention-internal reduction of QK^T); [KB] "计算 attention score 时".
    Softmax and the value product are the ordinary ones: a selection of P's
    columns would need P whole before the product, so only the score product is
    reduced here.  Q [B, Hq, nq, dh], K / V [B, Hkv, nk, dh] -> O [B, Hq, nq, dh], I.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Bsz, hq, nq, dh = Q.shape
    hkv = K.shape[1]
    k = retention_count(rho, dh)
    O = np.empty((Bsz, hq, nq, V.shape[3]))
    I = np.empty((Bsz, hq, k), dtype=np.int64)
    for b in range(Bsz):
        for h in range(hq):
            g = kv_head(h, hq, hkv)
            O[b, h], I[b, h] = rmm_attention_rows(Q[b, h], K[b, g], V[b, g], rho, None, causal, scale)
    return {"O": O, "I": I}


def attention_rows(Qh: np.ndarray, Kg: np.ndarray, Vg: np.ndarray, I, rows=None, causal: bool = True,
                   scale: float = 1.0) -> np.ndarray:
    """Rows ``rows`` of one head's attention output with the reduced score product on
    a GIVEN index set I: softmax_rows(qk_scores_rows(...)) . Vg (see ``rmm_attention``).
    The row maximum is subtracted before exponentiating (it cancels in the ratio)."""
    S = qk_scores_rows(Qh, Kg, I, rows, causal, scale)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=1, keepdims=True)
    return P @ np.asarray(Vg, dtype=np.float64)


def rmm_attention_rows(Qh, Kg, Vg, rho: float, rows=None, causal: bool = True, scale: float = 1.0, I=None):
    """Rows ``rows`` of one head of ``rmm_attention``: I = the oracle's TopK of Qh's
    column norms (or the given set), then ``attention_rows``.  Returns (O_rows, I)."""
    Qh = np.asarray(Qh, dtype=np.float64)
    if I is None:
        I = topk_ascending(column_norms(Qh), retention_count(rho, Qh.shape[1]))
    I = _check_index_set(I, Qh.shape[1], "attention")
    return attention_rows(Qh, Kg, Vg, I, rows, causal, scale), I
