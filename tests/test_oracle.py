"""Pins for the CPU oracle: it is checked against things other than itself.

Hand-derived fixtures (tests/golden/*.json, each with its citation), closed
forms, brute force over all subsets on tiny d, and invariants of the
mathematics.  Each check is chosen so that a plausible slip in the oracle (row
norms instead of column norms, the wrong tie rule, a dropped term, a transposed
or mismatched operand, the wrong GQA head, a causal mask off by one) fails.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import synthetic

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- k = ceil(rho d)
def test_retention_count_table():
    fx = load("retention_count.json")
    for rho, d, k in fx["cases"]:
        assert oracle.retention_count(rho, d) == k, (rho, d)
    for rho, d in fx["invalid"]:
        rho = float(rho)
        with pytest.raises(ValueError):
            oracle.retention_count(rho, d)


# ----------------------------------------------------------------- hand fixtures
def test_linear_hand_fixture():
    fx = load("linear_hand.json")
    A = np.array(fx["A"], float)
    B = np.array(fx["B"], float)
    assert np.array_equal(oracle.column_sq_norms(A), np.array(fx["colsq"], float))
    for case in fx["cases"]:
        out = oracle.rmm_linear(A, B, case["rho"])
        assert out["I"].tolist() == case["I"], case["rho"]
        assert len(out["I"]) == case["k"]
        assert out["retained"] == pytest.approx(case["retained_num"] / case["retained_den"], abs=1e-15)
        if "Y" in case:
            assert np.array_equal(out["Y"], np.array(case["Y"], float))
        if "err_fro_sq" in case:
            dense = np.array(fx["dense"], float)
            err = np.sum((dense - out["Y"]) ** 2)
            assert err == case["err_fro_sq"]
            bound = case["bound_int"] + case["bound_sqrt5"] * math.sqrt(5)
            assert oracle.error_bound(A, B, out["I"]) == pytest.approx(bound, rel=1e-14)


def test_qk_hand_fixture_and_gqa():
    fx = load("qk_hand.json")
    Q = np.array(fx["Q"], float)
    K = np.array(fx["K"], float)
    exp_c = np.array([[[np.nan if v is None else v for v in row] for row in h] for h in fx["S_causal"][0]])
    exp_f = np.array(fx["S_full"][0], float)
    out = oracle.rmm_qk(Q, K, fx["rho"], causal=True)
    assert out["I"].tolist() == fx["I"]
    S = out["S"][0]
    assert np.array_equal(np.isneginf(S), np.isnan(exp_c))
    fin = ~np.isnan(exp_c)
    assert np.array_equal(S[fin], exp_c[fin])
    full = oracle.rmm_qk(Q, K, fx["rho"], causal=False, scale=0.5)
    assert np.array_equal(full["S"][0], 0.5 * exp_f)
    # GQA: Hq = 4, Hkv = 2; query heads 2,3 repeat 0,1 and must read key head 1 = 10 K.
    f = fx["gqa_key_head1_factor"]
    Q4 = np.concatenate([Q, Q], axis=1)
    K2 = np.concatenate([K, f * K], axis=1)
    g = oracle.rmm_qk(Q4, K2, fx["rho"], causal=False)
    assert np.array_equal(g["S"][0, :2], exp_f)
    assert np.array_equal(g["S"][0, 2:], f * exp_f)
    assert [oracle.kv_head(h, 4, 2) for h in range(4)] == [0, 0, 1, 1]
    assert [oracle.kv_head(h, 32, 8) for h in (0, 3, 4, 31)] == [0, 0, 1, 7]


def test_pv_hand_fixture():
    fx = load("pv_hand.json")
    P = np.array(fx["P"], float)
    V = np.array(fx["V"], float)
    c = oracle.rmm_pv(P, V, fx["rho"], causal=True)
    assert c["I"][0, 0].tolist() == fx["causal"]["I"]
    assert np.array_equal(c["O"][0, 0], np.array(fx["causal"]["O"], float))
    assert np.array_equal(oracle.column_sq_norms(P[0, 0], causal=True), np.array(fx["causal"]["colsq"], float))
    nc = oracle.rmm_pv(P, V, fx["rho"], causal=False)
    assert nc["I"][0, 0].tolist() == fx["noncausal"]["I"]
    assert np.array_equal(nc["O"][0, 0], np.array(fx["noncausal"]["O"], float))


# ----------------------------------------------------------------- brute force
def _unit_columns(g, n, d):
    U = g.standard_normal((n, d))
    return U / np.sqrt(np.sum(U * U, axis=0))[None, :]


def test_topk_maximises_retained_mass_bruteforce_known_norms():
    """Theorem 1 in checkable form: over all |S| = k subsets, the chosen set has the
    largest retained column-norm mass sum_{j in S} s_j (and energy sum s_j^2).  The
    columns are built with known norms c_j (A[:, j] = c_j u_j, u_j unit), so the
    test does not recompute norms from A."""
    g = np.random.Generator(np.random.PCG64(7))
    d, k, n = 12, 6, 16
    subsets = np.array(list(itertools.combinations(range(d), k)))
    for _ in range(100):
        c = np.exp(g.standard_normal(d))
        A = _unit_columns(g, n, d) * c[None, :]
        I, _, _ = oracle.select(A, 0.5)
        mass = c[subsets].sum(axis=1)
        best = subsets[np.argmax(mass)]
        assert I.tolist() == best.tolist()
        assert c[I].sum() >= mass.max() * (1 - 1e-12)
        assert (c[I] ** 2).sum() >= (c[subsets] ** 2).sum(axis=1).max() * (1 - 1e-12)


def test_topk_bruteforce_with_ties_lexicographic():
    """Equal norms: the lexicographically smallest maximiser is chosen."""
    d, k = 12, 6
    c = np.array([3, 1, 3, 2, 3, 1, 2, 3, 2, 1, 3, 2], float)
    # exact column norms: column j is c_j times a basis vector (a permuted diagonal)
    A = np.zeros((d, d))
    A[(np.arange(d) * 5) % d, np.arange(d)] = c
    I, _, _ = oracle.select(A, 0.5)
    subsets = list(itertools.combinations(range(d), k))
    mass = [sum(c[list(s)]) for s in subsets]
    best = max(mass)
    first = min(s for s, m in zip(subsets, mass) if m == best)
    assert first == (0, 2, 3, 4, 7, 10)
    assert tuple(I.tolist()) == first


def test_row_norms_would_fail():
    """Rows and columns carry different norms: selecting on row norms (a transposed
    score) picks a different set than the known column norms."""
    A = np.array([[10.0, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0], [0, 0, 0, 2], [0, 9, 0, 0]])
    I, q, _ = oracle.select(A, 0.5)
    assert q.tolist() == [100.0, 82.0, 1.0, 4.0]
    assert I.tolist() == [0, 1]


def test_all_equal_norms_pick_prefix_and_k1_argmax():
    for d in (1, 5, 12, 64):
        A = np.ones((3, d))
        for rho in (0.25, 0.5, 1.0):
            k = oracle.retention_count(rho, d)
            I, _, _ = oracle.select(A, rho)
            assert I.tolist() == list(range(k))
    g = np.random.Generator(np.random.PCG64(11))
    for _ in range(20):
        A = g.standard_normal((5, 40))
        norms2 = [sum(A[i, j] ** 2 for i in range(5)) for j in range(40)]
        I, _, _ = oracle.select(A, 1e-6)
        assert I.tolist() == [int(np.argmax(norms2))]


def test_reduced_product_bruteforce_loops():
    """A[:, I] B[I, :] against explicit Python loops on tiny random inputs."""
    g = np.random.Generator(np.random.PCG64(5))
    for _ in range(25):
        n, d, m = g.integers(1, 6), g.integers(1, 9), g.integers(1, 6)
        A = g.standard_normal((n, d))
        B = g.standard_normal((d, m))
        k = int(g.integers(1, d + 1))
        I = np.sort(g.choice(d, size=k, replace=False))
        Y = oracle.reduced_product(A, B, I)
        for i in range(n):
            for c in range(m):
                ref = 0.0
                for j in I:
                    ref += A[i, j] * B[j, c]
                assert Y[i, c] == pytest.approx(ref, rel=1e-12, abs=1e-12)


def test_identity_weight_masks_columns():
    g = np.random.Generator(np.random.PCG64(9))
    A = g.standard_normal((7, 10)) * np.exp(g.standard_normal(10))[None, :]
    out = oracle.rmm_linear(A, np.eye(10), 0.4)
    expect = np.zeros_like(A)
    expect[:, out["I"]] = A[:, out["I"]]
    assert np.array_equal(out["Y"], expect)


def test_rho_one_is_the_dense_product_bruteforce():
    g = np.random.Generator(np.random.PCG64(13))
    A = g.standard_normal((4, 6))
    B = g.standard_normal((6, 3))
    Y = oracle.rmm_linear(A, B, 1.0)["Y"]
    for i in range(4):
        for c in range(3):
            assert Y[i, c] == pytest.approx(sum(A[i, j] * B[j, c] for j in range(6)), rel=1e-12)


def test_error_bound_holds_on_tiny_draws():
    for A, B in synthetic.tiny_bruteforce_set(draws=100):
        out = oracle.rmm_linear(A, B, 0.5)
        dense = np.array([[sum(A[i, j] * B[j, c] for j in range(A.shape[1])) for c in range(B.shape[1])]
                          for i in range(A.shape[0])])
        err = math.sqrt(float(np.sum((dense - out["Y"]) ** 2)))
        assert err <= oracle.error_bound(A, B, out["I"]) * (1 + 1e-12) + 1e-300


def test_nested_sets_monotone_energy_scale_invariance():
    g = np.random.Generator(np.random.PCG64(17))
    for _ in range(10):
        A = g.standard_normal((9, 33)) * np.exp(1.5 * g.standard_normal(33))[None, :]
        prev, prev_e = set(), 0.0
        for rho in (0.1, 0.3, 0.5, 0.7, 0.9, 1.0):
            I, _, e = oracle.select(A, rho)
            assert prev <= set(I.tolist())
            assert e >= prev_e - 1e-15
            prev, prev_e = set(I.tolist()), e
            I2, _, _ = oracle.select(A * 4.0, rho)
            assert np.array_equal(I, I2)
        assert prev_e == 1.0


def test_permutation_equivariance():
    g = np.random.Generator(np.random.PCG64(19))
    A = g.standard_normal((6, 20)) * np.exp(g.standard_normal(20))[None, :]
    B = g.standard_normal((20, 5))
    perm = g.permutation(20)
    a = oracle.rmm_linear(A, B, 0.5)
    b = oracle.rmm_linear(A[:, perm], B[perm, :], 0.5)
    assert sorted(perm[b["I"]].tolist()) == a["I"].tolist()
    assert np.allclose(a["Y"], b["Y"], rtol=1e-12, atol=1e-12)


def test_causal_alignment_bottom_right():
    Q = np.ones((1, 1, 2, 4))
    K = np.ones((1, 1, 5, 4))
    S = oracle.rmm_qk(Q, K, 1.0, causal=True)["S"][0, 0]
    # nq = 2, nk = 5: query i sees keys j <= i + 3
    assert np.isfinite(S).tolist() == [[True] * 4 + [False], [True] * 5]
    P = np.ones((1, 1, 2, 5))
    V = np.arange(10, dtype=float).reshape(1, 1, 5, 2)
    O = oracle.rmm_pv(P, V, 1.0, causal=True)["O"][0, 0]
    assert O.tolist() == [[0 + 2 + 4 + 6, 1 + 3 + 5 + 7], [20, 25]]


def test_near_tie_band():
    s = np.array([1.0, 2.0, 2.0 * (1 + 5e-6), 3.0, 2.0 * (1 - 2e-5)])
    band = oracle.near_tie_band(s, 3)
    assert band.tolist() == [1, 2]


def test_synthetic_generators_are_seeded_and_shaped():
    A, B = synthetic.linear_small()
    A2, _ = synthetic.linear_small()
    assert tuple(A.shape) == (128, 1024) and tuple(B.shape) == (1024, 1024)
    assert bool((A == A2).all())
    Q, K = synthetic.qk_inputs(hq=4, hkv=2, n=64)
    assert tuple(Q.shape) == (1, 4, 64, 128) and tuple(K.shape) == (1, 2, 64, 128)
    P, V = synthetic.pv_inputs(heads=2, n=64)
    Pw = synthetic.widen(P)
    assert np.allclose(Pw.sum(axis=-1), 1.0, atol=2e-2)
    assert np.all(np.triu(Pw[0, 0], 1) == 0)


# ----------------------------------------------------------------- decode attention
def test_decode_qk_hand_fixture_group_selection():
    fx = load("decode_hand.json")["qk"]
    Q = np.array(fx["Q"], dtype=np.float64)
    Kt = np.array(fx["Kt_dim_major"], dtype=np.float64)
    r = oracle.rmm_decode_qk(Q, Kt, fx["rho"])
    assert np.array_equal(r["I"], np.array(fx["I"]))
    assert np.allclose(r["S"], np.array(fx["S"]), rtol=0, atol=1e-12)
    dense = oracle.rmm_decode_qk(Q, Kt, 1.0)
    assert np.allclose(dense["S"], np.array(fx["S_dense"]), rtol=0, atol=1e-12)
    # a per-head selection (each head alone) gives other scores: the grouped reading is what is pinned
    per_head = oracle.rmm_decode_qk(Q.reshape(1, 2, 1, 4)[:, :, 0], np.repeat(Kt, 2, axis=1), fx["rho"])
    assert not np.allclose(per_head["S"], r["S"])


def test_decode_pv_hand_fixture_and_bound():
    fx = load("decode_hand.json")["pv"]
    P = np.array(fx["P"], dtype=np.float64)
    V = np.array(fx["V"], dtype=np.float64)
    r = oracle.rmm_decode_pv(P, V, fx["rho"])
    assert np.array_equal(r["I"], np.array(fx["I"]))
    assert np.allclose(r["O"], np.array(fx["O"]), rtol=0, atol=1e-12)
    dense = oracle.rmm_decode_pv(P, V, 1.0)
    assert np.allclose(dense["O"], np.array(fx["O_dense"]), rtol=0, atol=1e-12)
    err = np.linalg.norm(dense["O"] - r["O"])
    assert abs(err - fx["error"]) < 1e-3 and err <= fx["bound"]
    assert abs(oracle.error_bound(P[0], V[0, 0], r["I"][0, 0]) - fx["bound"]) < 1e-3


def test_decode_rho_one_is_the_dense_product_bruteforce():
    g = np.random.default_rng(7)
    B, hq, hkv, dh, L, nk = 2, 4, 2, 6, 9, 7
    Q = g.standard_normal((B, hq, dh))
    Kt = g.standard_normal((B, hkv, dh, L))
    P = g.random((B, hq, L))
    V = g.standard_normal((B, hkv, L, dh))
    S = oracle.rmm_decode_qk(Q, Kt, 1.0, scale=0.5, nk=nk)["S"]
    O = oracle.rmm_decode_pv(P, V, 1.0, nk=nk)["O"]
    for b in range(B):
        for h in range(hq):
            g_ = h // (hq // hkv)
            for j in range(nk):
                acc = 0.0
                for t in range(dh):
                    acc += Q[b, h, t] * Kt[b, g_, t, j]
                assert abs(S[b, h, j] - 0.5 * acc) < 1e-12
            for c in range(dh):
                acc = 0.0
                for j in range(nk):  # tokens at and beyond nk are not part of the cache
                    acc += P[b, h, j] * V[b, g_, j, c]
                assert abs(O[b, h, c] - acc) < 1e-12


def test_decode_group_of_one_keeps_the_largest_magnitudes():
    """Hq = Hkv: the column norm of a single row is |x_j|, so the kept set is the k
    largest |p_j| (QK: |q_t|), lower index first on ties."""
    g = np.random.default_rng(8)
    P = np.round(g.standard_normal((1, 3, 40)), 1)  # rounding makes ties
    V = g.standard_normal((1, 3, 40, 4))
    k = oracle.retention_count(0.3, 40)
    I = oracle.rmm_decode_pv(P, V, 0.3)["I"]
    for h in range(3):
        order = sorted(range(40), key=lambda j: (-abs(P[0, h, j]), j))
        assert list(I[0, h]) == sorted(order[:k])
    Q = np.round(g.standard_normal((1, 2, 16)), 1)
    Kt = g.standard_normal((1, 2, 16, 5))
    kq = oracle.retention_count(0.5, 16)
    Iq = oracle.rmm_decode_qk(Q, Kt, 0.5)["I"]
    for h in range(2):
        order = sorted(range(16), key=lambda t: (-abs(Q[0, h, t]), t))
        assert list(Iq[0, h]) == sorted(order[:kq])


def test_decode_error_bound_and_head_order_invariance():
    g = np.random.default_rng(9)
    for _ in range(20):
        Q = g.standard_normal((1, 4, 8)) * np.exp(g.standard_normal(8))
        Kt = g.standard_normal((1, 1, 8, 11))
        red = oracle.rmm_decode_qk(Q, Kt, 0.5)
        dense = oracle.rmm_decode_qk(Q, Kt, 1.0)["S"]
        I = red["I"][0, 0]
        # the pages' bound with A = the group's query rows and B = the kept cache rows
        assert np.linalg.norm(dense - red["S"]) <= oracle.error_bound(Q[0], Kt[0, 0], I) + 1e-9
        perm = g.permutation(4)
        assert np.array_equal(oracle.rmm_decode_qk(Q[:, perm], Kt, 0.5)["I"], red["I"])


# ----------------------------------------------------------------- MLP block
def test_mlp_hand_fixture():
    fx = load("mlp_hand.json")
    X, Wg, Wu, Wd = (np.array(fx[n], dtype=np.float64) for n in ("X", "Wg", "Wu", "Wd"))
    r = oracle.rmm_mlp(X, Wg, Wu, Wd, fx["rho_gu"], fx["rho_down"])
    assert list(r["I_gu"]) == fx["I_gu"] and list(r["I_down"]) == fx["I_down"]
    assert np.allclose(r["H"], np.array(fx["H"]), rtol=0, atol=1e-12)
    assert np.allclose(r["Y"], np.array(fx["Y"]), rtol=0, atol=1e-12)
    dense = oracle.rmm_mlp(X, Wg, Wu, Wd, 1.0, 1.0)
    assert np.allclose(dense["H"][1], np.array(fx["H_dense_row1"]), rtol=0, atol=1e-9)


def test_mlp_rho_one_is_the_dense_block_bruteforce():
    g = np.random.default_rng(10)
    n, d, f, m = 3, 5, 4, 3
    X, Wg, Wu, Wd = g.standard_normal((n, d)), g.standard_normal((d, f)), g.standard_normal((d, f)), g.standard_normal((f, m))
    r = oracle.rmm_mlp(X, Wg, Wu, Wd, 1.0, 1.0)
    for i in range(n):
        h = []
        for c in range(f):
            gs = sum(X[i, j] * Wg[j, c] for j in range(d))
            us = sum(X[i, j] * Wu[j, c] for j in range(d))
            h.append(gs / (1.0 + math.exp(-gs)) * us)
            assert abs(r["H"][i, c] - h[-1]) < 1e-12
        for c in range(m):
            assert abs(r["Y"][i, c] - sum(h[j] * Wd[j, c] for j in range(f))) < 1e-12


def test_mlp_gate_and_up_use_the_same_columns():
    """With identity gate and up weights, G = U = X with the dropped columns zeroed,
    so H = SiLU(x) x exactly on the kept columns of X and 0 on the others."""
    g = np.random.default_rng(11)
    X = g.standard_normal((4, 9)) * np.exp(g.standard_normal(9))
    r = oracle.rmm_mlp_gate_up(X, np.eye(9), np.eye(9), 0.5)
    I, _, _ = oracle.select(X, 0.5)
    assert np.array_equal(r["I"], I)
    keep = np.zeros(9, dtype=bool)
    keep[I] = True
    assert np.allclose(r["H"][:, keep], X[:, keep] ** 2 / (1.0 + np.exp(-X[:, keep])), rtol=1e-14, atol=0)
    assert not r["H"][:, ~keep].any()


def test_mlp_down_bound_and_silu_values():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.silu(np.array([40.0]))[0] - 40.0) < 1e-12 and abs(oracle.silu(np.array([-40.0]))[0]) < 1e-15
    g = np.random.default_rng(12)
    for _ in range(10):
        X, Wg, Wu, Wd = g.standard_normal((5, 8)), g.standard_normal((8, 6)), g.standard_normal((8, 6)), g.standard_normal((6, 4))
        r = oracle.rmm_mlp(X, Wg, Wu, Wd, 0.7, 0.5)
        assert np.linalg.norm(r["H"] @ Wd - r["Y"]) <= oracle.error_bound(r["H"], Wd, r["I_down"]) + 1e-9


# ----------------------------------------------------------------- int8 weights
def test_int8_hand_fixture():
    fx = load("int8_hand.json")
    r = oracle.rmm_linear_int8(np.array(fx["A"], float), np.array(fx["Wq"], float), np.array(fx["scale"]), fx["rho"])
    assert list(r["I"]) == fx["I"]
    assert np.allclose(r["Y"], np.array(fx["Y"]), rtol=0, atol=1e-12)


def test_int8_rho_one_bruteforce_and_scale_per_column():
    g = np.random.default_rng(13)
    A = g.integers(-4, 5, size=(3, 6)).astype(float)
    Wq = g.integers(-127, 128, size=(6, 5)).astype(float)
    s = g.random(5) + 0.1
    Y = oracle.rmm_linear_int8(A, Wq, s, 1.0)["Y"]
    for i in range(3):
        for c in range(5):
            assert abs(Y[i, c] - s[c] * sum(A[i, j] * Wq[j, c] for j in range(6))) < 1e-9
    # doubling one column's scale doubles that output column only
    s2 = s.copy()
    s2[2] *= 2.0
    Y2 = oracle.rmm_linear_int8(A, Wq, s2, 1.0)["Y"]
    assert np.allclose(Y2[:, 2], 2.0 * Y[:, 2]) and np.allclose(np.delete(Y2, 2, 1), np.delete(Y, 2, 1))


def test_int8_keeps_the_bf16_selection():
    """The index set depends on A only: the same I as the bf16 projection for any weights."""
    g = np.random.default_rng(14)
    A = g.standard_normal((4, 20)) * np.exp(g.standard_normal(20))
    Wq = g.integers(-127, 128, size=(20, 7)).astype(float)
    r = oracle.rmm_linear_int8(A, Wq, np.ones(7), 0.4)
    assert np.array_equal(r["I"], oracle.select(A, 0.4)[0])
    keep = np.zeros(20, bool)
    keep[r["I"]] = True
    assert np.allclose(r["Y"], A[:, keep] @ Wq[keep], rtol=1e-12, atol=1e-9)


# ----------------------------------------------------------------- fused reduced attention
def test_attention_hand_fixture():
    fx = load("attention_hand.json")
    Q, K, V = (np.array(fx[n], dtype=np.float64) for n in ("Q", "K", "V"))
    r = oracle.rmm_attention(Q, K, V, fx["rho"], causal=True, scale=fx["scale"])
    assert list(r["I"][0, 0]) == fx["I"]
    assert np.allclose(r["O"][0, 0], np.array(fx["O_causal"]), rtol=0, atol=1e-12)
    nc = oracle.rmm_attention(Q, K, V, fx["rho"], causal=False)
    assert np.allclose(nc["O"][0, 0, 0], fx["O_noncausal_row0"], rtol=0, atol=1e-12)
    dense = oracle.rmm_attention(Q, K, V, 1.0, causal=False)
    assert np.allclose(dense["O"][0, 0, 0], fx["O_dense_noncausal_row0"], rtol=0, atol=1e-12)


def test_attention_rho_one_bruteforce_gqa_causal():
    g = np.random.default_rng(15)
    B, hq, hkv, n, dh = 1, 4, 2, 5, 3
    Q, K, V = g.standard_normal((B, hq, n, dh)), g.standard_normal((B, hkv, n, dh)), g.standard_normal((B, hkv, n, dh))
    O = oracle.rmm_attention(Q, K, V, 1.0, causal=True, scale=0.7)["O"]
    for h in range(hq):
        gk = h // 2
        for i in range(n):
            sc = [0.7 * sum(Q[0, h, i, t] * K[0, gk, j, t] for t in range(dh)) for j in range(i + 1)]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            for c in range(dh):
                ref = sum(w[j] * V[0, gk, j, c] for j in range(i + 1)) / sum(w)
                assert abs(O[0, h, i, c] - ref) < 1e-12


def test_attention_rows_are_convex_combinations_and_first_row_is_v0():
    """Softmax weights are positive and sum to one, so each output row lies within
    the per-column range of the visible V rows; under a causal mask with nq = nk the
    first query sees only key 0."""
    g = np.random.default_rng(16)
    Q, K, V = g.standard_normal((1, 2, 9, 8)), g.standard_normal((1, 1, 9, 8)), g.standard_normal((1, 1, 9, 8))
    O = oracle.rmm_attention(Q, K, V, 0.5, causal=True)["O"]
    for h in range(2):
        assert np.allclose(O[0, h, 0], V[0, 0, 0], rtol=0, atol=1e-12)
        for i in range(9):
            lo, hi = V[0, 0, :i + 1].min(axis=0), V[0, 0, :i + 1].max(axis=0)
            assert np.all(O[0, h, i] >= lo - 1e-12) and np.all(O[0, h, i] <= hi + 1e-12)
    # the same index sets as the score product alone
    assert np.array_equal(oracle.rmm_attention(Q, K, V, 0.5)["I"], oracle.rmm_qk(Q, K, 0.5)["I"])


# ---------------------------------------------------------------- the helpers, each on its own
def test_column_norms_pythagorean_columns_and_causal_mask():
    """Columns (3, 4), (5, 12) and (8, 15) have norms 5, 13 and 17; under a causal
    mask with nq = nk = 2, entry (0, 1) is not visible, so column 1's norm is 12."""
    A = np.array([[3.0, 5.0, 8.0], [4.0, 12.0, 15.0]])
    assert oracle.column_norms(A).tolist() == [5.0, 13.0, 17.0]
    Ac = np.array([[3.0, 99.0], [4.0, 12.0]])  # 99 sits above the diagonal
    assert oracle.column_norms(Ac, causal=True).tolist() == [5.0, 12.0]


def test_topk_ascending_order_ties_and_bounds():
    s = np.array([2.0, 7.0, 7.0, 1.0, 7.0, 0.0])
    assert oracle.topk_ascending(s, 1).tolist() == [1]        # three-way tie: the lowest index
    assert oracle.topk_ascending(s, 2).tolist() == [1, 2]
    assert oracle.topk_ascending(s, 4).tolist() == [0, 1, 2, 4]
    assert oracle.topk_ascending(s, 6).tolist() == [0, 1, 2, 3, 4, 5]
    with pytest.raises(ValueError):
        oracle.topk_ascending(s, 0)
    with pytest.raises(ValueError):
        oracle.topk_ascending(s, 7)


def test_retained_energy_closed_form():
    q = np.array([1.0, 4.0, 9.0, 16.0])  # squared norms of columns with norms 1..4
    assert oracle.retained_energy(q, np.array([2, 3])) == 25.0 / 30.0
    assert oracle.retained_energy(q, np.arange(4)) == 1.0
    assert oracle.retained_energy(np.zeros(3), np.array([0])) == 1.0  # nothing to lose


def test_linear_rows_hand_example():
    """A = [[1, 2], [3, 4]], B = identity, I = {1}: row 1 of A[:, I] B[I, :] is
    [0, 4] (column 0 of B is not used)."""
    A = np.array([[1.0, 2.0], [3.0, 4.0]])
    out = oracle.rmm_linear_rows(A, np.eye(2), np.array([1]), [1])
    assert out.tolist() == [[0.0, 4.0]]


def test_qk_and_pv_rows_match_the_full_products():
    """The row-sampled QK and PV restatements give exactly the rows of the full
    per-head products, with the same index sets (the full products are pinned by the
    hand fixtures and brute force above)."""
    g = np.random.default_rng(21)
    Q, K = g.standard_normal((1, 4, 7, 8)), g.standard_normal((1, 2, 7, 8))
    full = oracle.rmm_qk(Q, K, 0.5, causal=True, scale=0.3)
    rows = [0, 3, 6]
    for h in range(4):
        S, I = oracle.rmm_qk_rows(Q[0, h], K[0, oracle.kv_head(h, 4, 2)], 0.5, rows, causal=True, scale=0.3)
        assert np.array_equal(I, full["I"][0, h])
        assert np.array_equal(S, full["S"][0, h][rows])
    P = np.abs(g.standard_normal((1, 2, 6, 6)))
    V = g.standard_normal((1, 1, 6, 4))
    fullp = oracle.rmm_pv(P, V, 0.5, causal=True)
    for h in range(2):
        O, I, q = oracle.rmm_pv_rows(P[0, h], V[0, 0], 0.5, [1, 5], causal=True)
        assert np.array_equal(I, fullp["I"][0, h])
        assert np.array_equal(O, fullp["O"][0, h][[1, 5]])
        assert np.array_equal(q, oracle.column_sq_norms(P[0, h], causal=True))


def test_products_on_a_given_index_set_bruteforce_loops():
    """The index-set-given restatements (the references of the GPU parity checks when
    the library's set is used) against explicit Python loops, on a set that is NOT
    the TopK one, so that a function silently re-selecting would fail."""
    g = np.random.default_rng(22)
    nq, nk, dh = 5, 7, 6
    Qh, Kg, Vg = g.standard_normal((nq, dh)), g.standard_normal((nk, dh)), g.standard_normal((nk, 3))
    I = np.array([0, 2, 5])
    Qh[:, 1] *= 10.0  # column 1 dominates the norms, so TopK would keep it; I does not
    assert 1 in oracle.topk_ascending(oracle.column_norms(Qh), 3) and 1 not in I
    rows = [0, 2, 4]
    S = oracle.qk_scores_rows(Qh, Kg, I, rows, causal=True, scale=0.5)
    for a, i in enumerate(rows):
        for j in range(nk):
            if j > i + (nk - nq):
                assert S[a, j] == -np.inf
            else:
                ref = 0.5 * sum(Qh[i, t] * Kg[j, t] for t in I)
                assert abs(S[a, j] - ref) < 1e-12
    # attention on the given set: softmax over the visible keys, then V
    O = oracle.attention_rows(Qh, Kg, Vg, I, rows, causal=True, scale=0.5)
    for a, i in enumerate(rows):
        vis = range(i + (nk - nq) + 1)
        sc = [0.5 * sum(Qh[i, t] * Kg[j, t] for t in I) for j in vis]
        mx = max(sc)
        w = [math.exp(x - mx) for x in sc]
        for c in range(3):
            ref = sum(w[j] * Vg[j, c] for j in vis) / sum(w)
            assert abs(O[a, c] - ref) < 1e-12
    # PV on a given set of key positions: entries above the diagonal count as zero
    Ph = np.abs(g.standard_normal((nq, nk)))
    J = np.array([1, 3, 6])
    Opv = oracle.pv_output_rows(Ph, Vg, J, rows, causal=True)
    for a, i in enumerate(rows):
        for c in range(3):
            ref = sum(Ph[i, j] * Vg[j, c] for j in J if j <= i + (nk - nq))
            assert abs(Opv[a, c] - ref) < 1e-12
    # int8 codes with per-column scales, and the MLP gate/up on one shared set
    A = g.standard_normal((4, 6))
    Wq = g.integers(-127, 128, size=(6, 5)).astype(np.float64)
    sc8 = g.uniform(0.01, 0.1, 5)
    Y8 = oracle.int8_product_rows(A, Wq, sc8, I, [1, 3])
    Wg, Wu = g.standard_normal((6, 5)), g.standard_normal((6, 5))
    H = oracle.mlp_gate_up_rows(A, Wg, Wu, I, [1, 3])
    for a, i in enumerate([1, 3]):
        for c in range(5):
            assert abs(Y8[a, c] - sc8[c] * sum(A[i, t] * Wq[t, c] for t in I)) < 1e-12
            gte = sum(A[i, t] * Wg[t, c] for t in I)
            up = sum(A[i, t] * Wu[t, c] for t in I)
            assert abs(H[a, c] - gte / (1.0 + math.exp(-gte)) * up) < 1e-12


def test_row_functions_match_the_full_functions():
    """With no index set given, every row function reproduces exactly the rows of the
    full function it samples, with the same index set (the full functions are pinned
    by the hand fixtures and brute force above)."""
    g = np.random.default_rng(23)
    Q, K, V = g.standard_normal((1, 4, 9, 8)), g.standard_normal((1, 2, 9, 8)), g.standard_normal((1, 2, 9, 8))
    full = oracle.rmm_attention(Q, K, V, 0.5, causal=True, scale=0.4)
    for h in range(4):
        gk = oracle.kv_head(h, 4, 2)
        O, I = oracle.rmm_attention_rows(Q[0, h], K[0, gk], V[0, gk], 0.5, [0, 4, 8], causal=True, scale=0.4)
        assert np.array_equal(I, full["I"][0, h])
        assert np.array_equal(O, full["O"][0, h][[0, 4, 8]])
        O2, _ = oracle.rmm_attention_rows(Q[0, h], K[0, gk], V[0, gk], 0.5, [0, 4, 8], causal=True, scale=0.4, I=I)
        assert np.array_equal(O2, O)
    X = g.standard_normal((6, 10))
    Wg, Wu, Wq = g.standard_normal((10, 4)), g.standard_normal((10, 4)), g.integers(-127, 128, (10, 4))
    sc = g.uniform(0.01, 0.1, 4)
    gu = oracle.rmm_mlp_gate_up(X, Wg, Wu, 0.6)
    assert np.array_equal(oracle.mlp_gate_up_rows(X, Wg, Wu, gu["I"], [1, 5]), gu["H"][[1, 5]])
    i8 = oracle.rmm_linear_int8(X, Wq, sc, 0.6)
    assert np.array_equal(oracle.int8_product_rows(X, Wq, sc, i8["I"], [0, 2]), i8["Y"][[0, 2]])
    P = np.abs(g.standard_normal((1, 1, 8, 8)))
    fullp = oracle.rmm_pv(P, V[:, :1, :8], 0.5, causal=True)
    Oi, Ii, _ = oracle.rmm_pv_rows(P[0, 0], V[0, 0, :8], 0.5, [2, 7], causal=True, I=fullp["I"][0, 0])
    assert np.array_equal(Oi, fullp["O"][0, 0][[2, 7]]) and np.array_equal(Ii, fullp["I"][0, 0])


@pytest.mark.parametrize("bad", [[2, 1], [1, 1], [-1, 2], [0, 8], []])
def test_given_index_sets_must_be_ascending_and_in_range(bad):
    Qh, Kg = np.ones((3, 8)), np.ones((3, 8))
    with pytest.raises(ValueError):
        oracle.qk_scores_rows(Qh, Kg, np.array(bad, dtype=np.int64), None)
