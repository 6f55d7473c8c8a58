"""Pins for the CPU oracle: invariants, closed forms and exact rational brute force.

These run without a GPU.  Each test pins the oracle to something other than
itself, chosen so that a dropped term, a wrong sign or index, or a transposed
operand in ``oracle/gdn_oracle.py`` fails at least one of them.
"""
from fractions import Fraction
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- #
# helpers independent of the oracle
# --------------------------------------------------------------------------- #
def random_chunks(nc, k, d, seed, gate_scale=1.0):
    """Chunks drawn like the workloads (unit-norm keys, sigmoid beta, -softplus gates)."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((nc, k, d))
    K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((nc, k, d))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((nc, k))))
    lg = -np.log1p(np.exp(rng.standard_normal((nc, k)))) * gate_scale
    g = np.cumsum(lg, axis=-1)
    return K, V, beta, g, lg


def frac_matrix(a):
    return [[Fraction(float(x)) for x in row] for row in a]


def frac_matmul(X, Y):
    n, m, p = len(X), len(Y), len(Y[0])
    return [[sum((X[i][l] * Y[l][j] for l in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def frac_eye(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def frac_sub(X, Y):
    return [[a - b for a, b in zip(r, s)] for r, s in zip(X, Y)]


def frac_add(X, Y):
    return [[a + b for a, b in zip(r, s)] for r, s in zip(X, Y)]


def frac_gauss_jordan_inverse(M):
    """Inverse by Gauss-Jordan elimination with exact rationals (no triangular shortcut)."""
    n = len(M)
    aug = [list(r) + [Fraction(int(i == j)) for j in range(n)] for i, r in enumerate(M)]
    for c in range(n):
        p = next(r for r in range(c, n) if aug[r][c] != 0)
        aug[c], aug[p] = aug[p], aug[c]
        piv = aug[c][c]
        aug[c] = [x / piv for x in aug[c]]
        for r in range(n):
            if r != c and aug[r][c] != 0:
                f = aug[r][c]
                aug[r] = [x - f * y for x, y in zip(aug[r], aug[c])]
    return [r[n:] for r in aug]


def frac_to_np(X):
    return np.array([[float(x) for x in r] for r in X])


def load_golden(fname: str = "unit_lower_4x4.txt"):
    out, name, rows = {}, None, []
    with open(os.path.join(GOLDEN, fname)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) == 1 and not parts[0].lstrip("-").isdigit():
                name, rows = parts[0], []
                out[name] = rows
            else:
                rows.append([float(x) for x in parts])
    return {k: np.array(v) for k, v in out.items()}


# --------------------------------------------------------------------------- #
# golden hand-derived example
# --------------------------------------------------------------------------- #
def test_golden_4x4_closed_forms():
    G = load_golden()
    A = G["A"][None]
    np.testing.assert_array_equal(O.invert_fwdsub(A)[0], G["T_exact"])
    np.testing.assert_array_equal(O.neumann_powers_sum(A, 3)[0], G["T_exact"])
    np.testing.assert_array_equal((A @ A)[0], G["A2"])
    np.testing.assert_array_equal(O.invert_neumann(A, 1, False, 0)[0], G["T0_N1_nomask"])
    np.testing.assert_array_equal(O.invert_neumann(A, 1, True, 0)[0], G["T0_N1_mask"])
    np.testing.assert_array_equal(O.invert_neumann(A, 2, False, 0)[0], G["T0_N2_nomask"])
    np.testing.assert_array_equal(O.invert_neumann(A, 2, True, 0)[0], G["T0_N2_mask"])
    T0 = O.invert_neumann(A, 1, True, 0)
    np.testing.assert_array_equal(O.residual_matrix(A, T0)[0], G["E_N1_mask"])
    np.testing.assert_array_equal(O.invert_neumann(A, 1, True, 1)[0], G["T_N1_mask_S1"])


def test_closed_form_2x2_3x3():
    a21, a31, a32 = 0.3, -0.7, 1.9
    A2 = np.array([[[0, 0], [a21, 0]]], float)
    np.testing.assert_allclose(O.invert_fwdsub(A2)[0], [[1, 0], [a21, 1]], rtol=0, atol=1e-15)
    A3 = np.array([[[0, 0, 0], [a21, 0, 0], [a31, a32, 0]]], float)
    T3 = O.invert_fwdsub(A3)[0]
    np.testing.assert_allclose(T3[2, 0], a31 + a32 * a21, rtol=1e-15)
    np.testing.assert_allclose(T3[2, 1], a32, rtol=1e-15)
    # Neumann N=1 is I + A: it misses only the a32*a21 path
    T0 = O.invert_neumann(A3, 1, False, 0)[0]
    np.testing.assert_allclose(T3 - T0, [[0, 0, 0], [0, 0, 0], [a32 * a21, 0, 0]], atol=1e-15)


def test_band_mask_definition():
    M = O.band_mask(6, 2)
    for i in range(6):
        for j in range(6):
            assert M[i, j] == (1.0 if i - j <= 2 else 0.0)


# --------------------------------------------------------------------------- #
# A
# --------------------------------------------------------------------------- #
def test_build_A_structure_and_no_overflow():
    K, _, beta, g, _ = random_chunks(3, 16, 8, seed=1)
    A = O.build_A(K, beta, g)
    assert np.all(np.triu(A) == 0.0)                       # strictly lower
    assert np.all(A[np.tril(np.ones((16, 16), bool), -1)[None].repeat(3, 0)] != 0.0)
    # a huge positive g_i - g_j above the diagonal must not reach exp
    g2 = np.tile(-1000.0 * np.arange(16.0), (3, 1))
    A2 = O.build_A(K, beta, g2)
    assert np.all(np.isfinite(A2))


def test_build_A_entry_by_entry_small():
    """Entry (i,j) against an explicit scalar loop with math.exp (3 tokens)."""
    K, _, beta, g, _ = random_chunks(1, 3, 4, seed=2)
    A = O.build_A(K, beta, g)[0]
    for i in range(3):
        for j in range(3):
            if i > j:
                dot = math.fsum(K[0, i, t] * K[0, j, t] for t in range(4))
                want = -beta[0, i] * dot * math.exp(g[0, i] - g[0, j])
                assert A[i, j] == pytest.approx(want, rel=1e-14)
            else:
                assert A[i, j] == 0.0


# --------------------------------------------------------------------------- #
# exact inverse and Lemma 3.1
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("k", [8, 64, 256])
def test_I1_fwdsub_is_inverse(k):
    K, _, beta, g, _ = random_chunks(4, k, 32, seed=k)
    A = O.build_A(K, beta, g)
    T = O.invert_fwdsub(A)
    R = (np.eye(k) - A) @ T
    assert np.abs(R - np.eye(k)).max() <= 1e-13 * max(1.0, np.abs(T).max())


@pytest.mark.parametrize("k", [4, 8])
def test_I6_bruteforce_rational(k):
    """fwdsub, the full series, T0 and the residual against exact rationals."""
    K, _, beta, g, _ = random_chunks(1, k, 5, seed=10 + k, gate_scale=0.1)
    A = O.build_A(K, beta, g)
    Af = frac_matrix(A[0])
    I = frac_eye(k)
    Tf = frac_gauss_jordan_inverse(frac_sub(I, Af))
    T = frac_to_np(Tf)
    np.testing.assert_allclose(O.invert_fwdsub(A)[0], T, rtol=1e-15, atol=1e-15)
    # truncated series with mask, then the residual correction (exact rationals)
    N, S = 1, 2
    P, T0f = I, I
    for _ in range(N):
        P = frac_matmul(P, Af)
        T0f = frac_add(T0f, P)
    T0f = [[x if i - j <= N else Fraction(0) for j, x in enumerate(r)] for i, r in enumerate(T0f)]
    Ef = frac_sub(I, frac_matmul(frac_sub(I, Af), T0f))
    acc, Ep = I, I
    for _ in range(S):
        Ep = frac_matmul(Ep, Ef)
        acc = frac_add(acc, Ep)
    Tres = frac_to_np(frac_matmul(T0f, acc))
    np.testing.assert_allclose(O.invert_neumann(A, N, True, 0)[0], frac_to_np(T0f),
                               rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(O.residual_matrix(A, O.invert_neumann(A, N, True, 0))[0],
                               frac_to_np(Ef), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(O.invert_neumann(A, N, True, S)[0], Tres, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("k", [16, 64])
def test_I2_lemma_3_1_powers_vanish(k):
    K, _, beta, g, _ = random_chunks(2, k, 16, seed=3)
    A = O.build_A(K, beta, g)
    i = np.arange(k)[:, None]
    j = np.arange(k)[None, :]
    P = np.broadcast_to(np.eye(k), A.shape).copy()
    for n in range(1, k + 1):
        P = P @ A
        assert np.all(P[:, (i - j) < n] == 0.0), n          # exact zeros
    assert np.all(P == 0.0)                                  # A^k = 0


@pytest.mark.parametrize("k", [16, 64])
def test_I3_full_series_is_exact(k):
    K, _, beta, g, _ = random_chunks(2, k, 32, seed=4, gate_scale=0.2)
    A = O.build_A(K, beta, g)
    T = O.invert_fwdsub(A)
    T_full = O.invert_neumann(A, k - 1, False, 0)
    assert O.rel_fro(T_full, T) <= 1e-12


@pytest.mark.parametrize("N", [1, 2, 3, 4])
def test_I4_band_equality(N):
    k = 64
    K, _, beta, g, _ = random_chunks(3, k, 64, seed=5, gate_scale=0.2)
    A = O.build_A(K, beta, g)
    T = O.invert_fwdsub(A)
    dist = np.arange(k)[:, None] - np.arange(k)[None, :]
    band = dist <= N
    for mask in (False, True):
        T0 = O.invert_neumann(A, N, mask, 0)
        err = np.abs(T0 - T)[:, band].max()
        assert err <= 1e-13 * np.abs(T).max()
        if mask:
            assert np.all(T0[:, ~band] == 0.0)
        else:
            # outside the band, the unmasked truncation differs from T
            assert np.abs(T0 - T)[:, dist == N + 1].max() > 0


@pytest.mark.parametrize("N,S", [(1, 1), (3, 1), (3, 8), (2, 3)])
def test_I5_residual_band_law(N, S):
    k = 64
    K, _, beta, g, _ = random_chunks(2, k, 64, seed=6, gate_scale=0.2)
    A = O.build_A(K, beta, g)
    T = O.invert_fwdsub(A)
    L = (S + 1) * (N + 1)
    dist = np.arange(k)[:, None] - np.arange(k)[None, :]
    scale = np.abs(T).max()
    for mask in (False, True):
        Tr = O.invert_neumann(A, N, mask, S)
        assert np.abs(Tr - T)[:, dist <= L - 1].max() <= 1e-12 * scale
        if L >= k:
            assert O.rel_fro(Tr, T) <= 1e-12
        else:
            assert np.abs(Tr - T)[:, dist == L].max() > 0
    # without the mask E = A^{N+1}, so the result is the Neumann series of order L-1
    Tr = O.invert_neumann(A, N, False, S)
    assert O.rel_fro(Tr, O.invert_neumann(A, L - 1, False, 0)) <= 1e-12
    E = O.residual_matrix(A, O.invert_neumann(A, N, False, 0))
    Ap = np.linalg.matrix_power(A, N + 1)
    assert np.abs(E - Ap).max() <= 1e-13


# --------------------------------------------------------------------------- #
# WY
# --------------------------------------------------------------------------- #
def test_I7_wy_triangular_solve_identity():
    k, d = 64, 32
    K, V, beta, g, _ = random_chunks(3, k, d, seed=7)
    A = O.build_A(K, beta, g)
    T = O.invert_fwdsub(A)
    W, U = O.wy(T, K, V, beta)
    I_A = np.eye(k) - A
    np.testing.assert_allclose(I_A @ W, beta[..., None] * K, atol=1e-12)
    np.testing.assert_allclose(I_A @ U, beta[..., None] * V, atol=1e-12)
    Wg, U2 = O.wy(T, K, V, beta, g)
    np.testing.assert_allclose(I_A @ Wg, (beta * np.exp(g))[..., None] * K, atol=1e-12)
    np.testing.assert_array_equal(U, U2)


def test_wy_rows_small_explicit():
    """W row i = sum_j T_ij beta_j k_j, explicit loop on a 3x3 chunk."""
    K, V, beta, g, _ = random_chunks(1, 3, 2, seed=8)
    T = np.array([[[1.0, 0, 0], [0.5, 1.0, 0], [-0.25, 2.0, 1.0]]])
    W, U = O.wy(T, K, V, beta)
    for i in range(3):
        for t in range(2):
            w = math.fsum(T[0, i, j] * beta[0, j] * K[0, j, t] for j in range(3))
            u = math.fsum(T[0, i, j] * beta[0, j] * V[0, j, t] for j in range(3))
            assert W[0, i, t] == pytest.approx(w, rel=1e-14)
            assert U[0, i, t] == pytest.approx(u, rel=1e-14)


# --------------------------------------------------------------------------- #
# full chunk-wise forward vs the token recurrence
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("T_len,d", [(256, 32), (1024, 128)])
def test_I8_chunk_form_equals_token_recurrence(T_len, d):
    k, BH = 64, 2
    rng = np.random.default_rng(9)
    K, V, beta, _, lg = random_chunks(BH * T_len // k, k, d, seed=9)
    K = K.reshape(BH, T_len, d)
    V = V.reshape(BH, T_len, d)
    beta = beta.reshape(BH, T_len)
    lg = lg.reshape(BH, T_len)
    Q = rng.standard_normal((BH, T_len, d))
    Q /= np.linalg.norm(Q, axis=-1, keepdims=True)
    S0 = 0.1 * rng.standard_normal((BH, d, d))
    n = T_len // k
    g = np.cumsum(lg.reshape(BH, n, k), axis=-1)
    Kc, Vc, Qc, bc = (x.reshape(BH, n, k, -1) for x in (K, V, Q, beta[..., None]))
    bc = bc[..., 0]
    A = O.build_A(Kc, bc, g)
    T = O.invert_fwdsub(A)
    Oc, Sc = O.chunk_forward(Qc, Kc, Vc, bc, g, T, S0)
    Ot, St = O.token_recurrence(Q, K, V, beta, lg, S0)
    assert O.rel_fro(Oc.reshape(BH, T_len, d), Ot) <= 1e-10
    assert O.rel_fro(Sc, St) <= 1e-10


# --------------------------------------------------------------------------- #
# prologue: normalised keys, chunk-local cumulative gates
# --------------------------------------------------------------------------- #
def test_l2_normalize_rows():
    x = np.array([[3.0, 4.0], [0.0, 0.0], [-1.0, 0.0]])
    assert np.array_equal(O.l2_normalize_rows(x), np.array([[0.6, 0.8], [0.0, 0.0], [-1.0, 0.0]]))
    rng = np.random.default_rng(41)
    K = rng.standard_normal((3, 5, 16)) * rng.uniform(0.1, 10.0, (3, 5, 1))
    Kn = O.l2_normalize_rows(K)
    assert np.allclose(np.linalg.norm(Kn, axis=-1), 1.0, rtol=0, atol=1e-15)
    assert np.allclose(Kn * np.linalg.norm(K, axis=-1, keepdims=True), K, rtol=1e-14, atol=0)


def test_chunk_cumsum_restarts_every_chunk():
    lg = np.arange(1.0, 9.0)[None]                    # 1..8, chunks of 4
    assert np.array_equal(O.chunk_cumsum(lg, 4), np.array([[1, 3, 6, 10, 5, 11, 18, 26.0]]))
    rng = np.random.default_rng(42)
    x = -rng.uniform(0, 1, (2, 3, 64))
    g = O.chunk_cumsum(x, 16)
    c = g.reshape(2, 3, 4, 16)
    assert np.allclose(np.diff(c, axis=-1), x.reshape(2, 3, 4, 16)[..., 1:], rtol=0, atol=1e-15)
    assert np.array_equal(c[..., 0], x.reshape(2, 3, 4, 16)[..., 0])


# --------------------------------------------------------------------------- #
# block-decomposition inverse (the other comparison point)
# --------------------------------------------------------------------------- #
def test_blocked_inverse_is_exact():
    K, _, beta, g, _ = random_chunks(3, 64, 32, seed=34)
    A = O.build_A(K, beta, g)
    for base in (16, 8, 4):
        T = O.invert_blocked(A, base)
        assert np.allclose((np.eye(64) - A) @ T, np.eye(64), rtol=0, atol=1e-13)
        assert np.allclose(T, O.invert_fwdsub(A), rtol=0, atol=1e-13)


def test_blocked_inverse_exact_rationals_4x4():
    """base 1 on a 4 x 4 chunk: every step is the 2 x 2 block formula; checked
    against the exact rational inverse."""
    rng = np.random.default_rng(35)
    A = np.tril(rng.integers(-4, 5, (4, 4)), -1).astype(np.float64) / 4.0
    T = O.invert_blocked(A[None], 1)[0]
    L = frac_matrix(np.eye(4) - A)
    # exact inverse of the unit lower-triangular L by forward substitution in rationals
    Tq = [[Fraction(int(i == j)) for j in range(4)] for i in range(4)]
    for i in range(4):
        for j in range(i):
            Tq[i][j] = -sum((L[i][l] * Tq[l][j] for l in range(j, i)), Fraction(0))
    assert all(Fraction(float(T[i][j])) == Tq[i][j] for i in range(4) for j in range(4))


# --------------------------------------------------------------------------- #
# sequential correction (the comparison point of the parallel residual)
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("N,mask", [(1, True), (3, True), (3, False), (2, True)])
def test_newton_steps_equal_parallel_residual_with_doubled_terms(N, mask):
    """M sequential steps sum 2^M terms of the residual series: with R_m the
    residual of T_m, R_{m+1} = R_m^2, so T_M = T0 (I + E + ... + E^(2^M - 1))."""
    K, _, beta, g, _ = random_chunks(3, 16, 8, seed=31)
    A = O.build_A(K, beta, g)
    for M in range(4):
        TN = O.invert_newton(A, N, mask, M)
        TP = O.invert_neumann(A, N, mask, 2 ** M - 1)
        assert np.allclose(TN, TP, rtol=0, atol=1e-12)


def test_newton_residual_squares_each_step():
    K, _, beta, g, _ = random_chunks(2, 16, 8, seed=32)
    A = O.build_A(K, beta, g)
    eye = np.eye(16)
    prev = O.residual_matrix(A, O.invert_newton(A, 2, True, 0))
    for M in range(1, 4):
        R = eye - (eye - A) @ O.invert_newton(A, 2, True, M)
        assert np.allclose(R, prev @ prev, rtol=0, atol=1e-13)
        prev = R


def test_newton_reaches_the_exact_inverse():
    """2^M (N + 1) >= k: the residual's power vanishes, T_M is exact."""
    K, _, beta, g, _ = random_chunks(2, 16, 8, seed=33)
    A = O.build_A(K, beta, g)
    T = O.invert_newton(A, 3, True, 2)                 # 4 * 4 >= 16
    assert np.allclose((np.eye(16) - A) @ T, np.eye(16), rtol=0, atol=1e-13)
    T1 = O.invert_newton(A, 3, True, 1)                # 2 * 4 < 16: not exact
    assert not np.allclose((np.eye(16) - A) @ T1, np.eye(16), rtol=0, atol=1e-9)


# --------------------------------------------------------------------------- #
# decode steps (grouped query/key heads)
# --------------------------------------------------------------------------- #
def test_decode_two_dim_closed_form():
    """One step by hand: S = I, k = e_1, v = (2, 3), b = 1/2, a = e^-1, q = (1, 1):
    S' = a (I - k k^T / 2) + v k^T / 2 = [[a/2 + 1, 0], [3/2, a]]."""
    a = math.exp(-1.0)
    Q = np.array([[[[1.0, 1.0]]]])
    K = np.array([[[[1.0, 0.0]]]])
    V = np.array([[[[2.0, 3.0]]]])
    Ob, Sb = O.decode(Q, K, V, np.full((1, 1, 1), 0.5), np.full((1, 1, 1), -1.0),
                      np.eye(2)[None, None])
    S_ref = np.array([[a / 2 + 1.0, 0.0], [1.5, a]])
    assert np.allclose(Sb[0, 0], S_ref, rtol=0, atol=1e-15)
    assert np.allclose(Ob[0, 0, 0], S_ref @ np.array([1.0, 1.0]), rtol=0, atol=1e-15)


def test_decode_full_write_retrieves_value():
    """Delta-rule property: with a = 1, b = 1 and a unit key, the updated state
    maps that key exactly onto its value (S' k = S k - S k + v)."""
    rng = np.random.default_rng(21)
    d = 16
    k = rng.standard_normal(d)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(d)
    S0 = rng.standard_normal((1, 1, d, d))
    _, S1 = O.decode(rng.standard_normal((1, 1, 1, d)), k[None, None, None], v[None, None, None],
                     np.ones((1, 1, 1)), np.zeros((1, 1, 1)), S0)
    assert np.allclose(S1[0, 0] @ k, v, rtol=0, atol=1e-12)


def test_decode_zero_beta_only_decays():
    rng = np.random.default_rng(22)
    d, n = 8, 3
    S0 = rng.standard_normal((1, 2, d, d))
    Q = rng.standard_normal((1, 1, n, d))
    lg = -np.abs(rng.standard_normal((1, 2, n)))
    Ob, Sb = O.decode(Q, rng.standard_normal((1, 1, n, d)), rng.standard_normal((1, 2, n, d)),
                      np.zeros((1, 2, n)), lg, S0)
    for h in range(2):
        decay = np.exp(np.cumsum(lg[0, h]))
        for t in range(n):
            assert np.allclose(Ob[0, h, t], decay[t] * S0[0, h] @ Q[0, 0, t], rtol=1e-13, atol=0)
        assert np.allclose(Sb[0, h], decay[-1] * S0[0, h], rtol=1e-13, atol=0)


def test_decode_equals_chunk_form():
    """Decoding 128 tokens one at a time equals the chunk-wise forward with the
    exact inverse (pinned above against the token recurrence)."""
    k, n, d, H = 64, 128, 32, 2
    rng = np.random.default_rng(23)
    K, V, beta, _, lg = random_chunks(H * n // k, k, d, seed=23)
    K, V = K.reshape(1, H, n, d), V.reshape(1, H, n, d)
    beta, lg = beta.reshape(1, H, n), lg.reshape(1, H, n)
    Q = rng.standard_normal((1, H, n, d))
    Q /= np.linalg.norm(Q, axis=-1, keepdims=True)
    S0 = 0.1 * rng.standard_normal((1, H, d, d))
    Od, Sd = O.decode(Q, K, V, beta, lg, S0)
    c = n // k
    g = np.cumsum(lg.reshape(H, c, k), axis=-1)
    Kc, Vc, Qc = (x.reshape(H, c, k, d) for x in (K, V, Q))
    bc = beta.reshape(H, c, k)
    T = O.invert_fwdsub(O.build_A(Kc, bc, g))
    Oc, Sc = O.chunk_forward(Qc, Kc, Vc, bc, g, T, S0[0])
    assert O.rel_fro(Od[0], Oc.reshape(H, n, d)) <= 1e-10
    assert O.rel_fro(Sd[0], Sc) <= 1e-10


def test_decode_value_heads_share_query_key_in_groups():
    """Hv = 2 Hk: value heads 2j and 2j + 1 read query/key head j, i.e. the same
    result as repeating each query/key head twice along the head axis."""
    rng = np.random.default_rng(24)
    B, Hk, Hv, n, d = 2, 2, 4, 3, 8
    Q = rng.standard_normal((B, Hk, n, d))
    K = rng.standard_normal((B, Hk, n, d))
    K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((B, Hv, n, d))
    beta = rng.uniform(0.1, 0.9, (B, Hv, n))
    lg = -rng.uniform(0.0, 1.0, (B, Hv, n))
    S0 = rng.standard_normal((B, Hv, d, d))
    Og, Sg = O.decode(Q, K, V, beta, lg, S0)
    Or, Sr = O.decode(np.repeat(Q, 2, axis=1), np.repeat(K, 2, axis=1), V, beta, lg, S0)
    assert np.array_equal(Og, Or) and np.array_equal(Sg, Sr)
    # and not the interleaved assignment h % Hk
    Oi, _ = O.decode(np.tile(Q, (1, 2, 1, 1)), np.tile(K, (1, 2, 1, 1)), V, beta, lg, S0)
    assert not np.allclose(Og, Oi)


# --------------------------------------------------------------------------- #
# INT8 scheme
# --------------------------------------------------------------------------- #
def test_I9_int8_codes_and_accumulators():
    k, N = 16, 3
    K, _, beta, g, _ = random_chunks(4, k, 16, seed=11, gate_scale=0.2)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    dist = np.arange(k)[:, None] - np.arange(k)[None, :]
    for mask in (False, True):
        r = O.int8_neumann(A32, N, mask)
        q, acc = r["q"], r["acc"]
        assert q.min() >= -127 and q.max() <= 127
        assert np.any(np.abs(q[:, 0]) == 127)               # amax maps to +-127
        for n in range(1, N):
            for c in range(4):
                for i in range(k):
                    for j in range(k):
                        want = sum(int(q[c, n - 1, i, l]) * int(q[c, 0, l, j]) for l in range(k))
                        if mask and dist[i, j] > N:
                            want = 0
                        assert int(acc[c, n, i, j]) == want
        if mask:
            assert np.all(q[:, :, dist > N] == 0)
            assert np.all(r["T"][:, dist > N] == 0)


def test_int8_rounding_half_even_and_scale():
    # amax = 127 gives r = 1 exactly, so the codes are rint of the entries
    A = np.zeros((1, 4, 4), np.float32)
    A[0, 1, 0] = 127.0
    A[0, 2, 0] = 2.5
    A[0, 2, 1] = -1.5
    A[0, 3, 0] = 0.5
    A[0, 3, 2] = 3.5
    r = O.int8_neumann(A, 1, False)
    assert r["q"][0, 0, 1, 0] == 127
    assert r["q"][0, 0, 2, 0] == 2      # half to even
    assert r["q"][0, 0, 2, 1] == -2
    assert r["q"][0, 0, 3, 0] == 0
    assert r["q"][0, 0, 3, 2] == 4
    assert r["scale"][0, 0] == np.float32(1.0)


def test_int8_scale_recursion_exact_integers():
    """Integer A with max 127: q_1 = A, s_1 = 1, and s_2 q_2 approximates A^2."""
    rng = np.random.default_rng(12)
    k = 8
    A = np.tril(rng.integers(-127, 128, (1, k, k)), -1).astype(np.float32)
    A[0, 1, 0] = 127.0
    r = O.int8_neumann(A, 2, False)
    np.testing.assert_array_equal(r["q"][0, 0], A[0].astype(np.int8))
    A2 = (A[0].astype(np.int64) @ A[0].astype(np.int64))
    m = np.abs(A2).max()
    assert r["scale"][0, 1] == np.float32(np.float32(m) / np.float32(127.0))
    # dequantised power within half a code step of the exact A^2
    deq = r["scale"][0, 1] * r["q"][0, 1].astype(np.float64)
    assert np.abs(deq - A2).max() <= 0.5 * m / 127 * (1 + 1e-6)
    # and the dequantised T is I + A + (that)
    np.testing.assert_allclose(r["T"][0], np.eye(k) + A[0] + deq, rtol=1e-6, atol=1e-3)


def test_int8_residual_tracks_the_float_formula_and_repairs_t0():
    """The int8 residual against the same correction in float64 on the same
    int8 T0 (E = I - (I - A) T0 and T0 sum E^s, literal powers): they differ
    only by the quantisation of A X, E and its powers, and X Gm.  Both beat
    the INT8 series alone by far (the pages' claim for N = 3, S = 8)."""
    K, _, beta, g, _ = random_chunks(8, 64, 128, seed=16)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    A64 = A32.astype(np.float64)
    exact = O.invert_fwdsub(A64)
    T0 = O.int8_neumann(A32, 3, True)["T"].astype(np.float64)
    E = np.eye(64) - (np.eye(64) - A64) @ T0
    for S in (1, 2, 8):
        acc = np.broadcast_to(np.eye(64), E.shape).copy()
        P = acc.copy()
        for _ in range(S):
            P = P @ E
            acc = acc + P
        Tf = T0 @ acc
        Tq = O.int8_residual(A32, 3, True, S)
        assert O.rel_fro(Tq, Tf) <= 5e-4
        assert O.rel_fro(Tq, exact) <= O.rel_fro(T0, exact) / 10
        assert np.all(np.triu(Tq, 1) == 0) and np.all(np.diagonal(Tq, axis1=1, axis2=2) == 1)


def test_int16_residual_tracks_the_float_formula_and_repairs_t0():
    """The int16 residual against the same correction in float64 on the same
    int16 T0 (literal powers of E = I - (I - A) T0): they differ only by the
    16-bit quantisation of A X, E and its powers, and X Gm.  It repairs the
    INT16 series by orders of magnitude, reaches the exact inverse within the
    codes' resolution, and stays far closer than the INT8 residual."""
    K, _, beta, g, _ = random_chunks(8, 64, 128, seed=16)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    A64 = A32.astype(np.float64)
    exact = O.invert_fwdsub(A64)
    r16 = O.int16_neumann(A32, 3, True)
    T0 = np.broadcast_to(np.eye(64), exact.shape).copy()
    for n in range(3):
        T0 = T0 + r16["scale"][:, n, None, None] * r16["q"][:, n].astype(np.float64)
    E = np.eye(64) - (np.eye(64) - A64) @ T0
    for S in (1, 2, 8):
        acc = np.broadcast_to(np.eye(64), E.shape).copy()
        P = acc.copy()
        for _ in range(S):
            P = P @ E
            acc = acc + P
        Tf = T0 @ acc
        Tq = O.int16_residual(A32, 3, True, S)
        assert Tq.dtype == np.float32
        assert O.rel_fro(Tq, Tf) <= 1e-5
        assert O.rel_fro(Tq, exact) <= O.rel_fro(r16["T"], exact) / 100
        if S == 8:          # truncation gone: only the codes' resolution is left
            assert O.rel_fro(Tq, exact) <= O.rel_fro(O.int8_residual(A32, 3, True, S), exact) / 20
        assert np.all(np.triu(Tq, 1) == 0) and np.all(np.diagonal(Tq, axis1=1, axis2=2) == 1)
    # a zero chunk: zero codes and scales everywhere, T = I exactly
    z = np.zeros((2, 8, 8), np.float32)
    assert np.array_equal(O.int16_residual(z, 3, True, 4), np.broadcast_to(np.eye(8, dtype=np.float32), z.shape))


def test_int8_residual_golden_by_hand():
    """The hand-derived INT8 example of tests/golden/int_residual_4x4.txt:
    E, its codes (one a tie, rounded to even), Gm and T exactly, for S = 1 and
    for S = 2, where E^2 has a zero maximum; and a matrix whose E is zero."""
    G = load_golden("int_residual_4x4.txt")
    A = G["A8"].astype(np.float32)[None]
    for S in (1, 2):
        r = O.int8_residual(A, 1, True, S, parts=True)
        assert np.array_equal(r["E"][0], G["E8"].astype(np.float32))
        assert np.array_equal(r["qE"][0], G["qE8"].astype(np.int64))
        assert r["sE"][0] == np.float32(2.0 ** -8)
        assert np.array_equal(r["Gm"][0], G["Gm8"].astype(np.float32))
        assert np.array_equal(r["qG"][0], G["qE8"].astype(np.int64)) and r["sG"][0] == np.float32(2.0 ** -8)
        assert np.array_equal(r["T"][0], G["T8"].astype(np.float32))
        assert np.array_equal(O.int8_residual(A, 1, True, S), r["T"])
    # one subdiagonal entry: X = A, A X = 0, so E = 0 (a zero maximum), T = I + A
    Z = np.zeros((1, 4, 4), np.float32)
    Z[0, 2, 1] = 0.5
    r = O.int8_residual(Z, 1, True, 3, parts=True)
    assert not r["E"].any() and not r["qE"].any() and r["sE"][0] == 0 and not r["Gm"].any()
    assert np.array_equal(r["T"][0], np.eye(4, dtype=np.float32) + Z[0])


def test_int16_residual_golden_by_hand():
    """The hand-derived INT16 example of tests/golden/int_residual_4x4.txt
    (binary64 scales, a tie at -2048.5, T rounded once to float32)."""
    G = load_golden("int_residual_4x4.txt")
    A = G["A16"].astype(np.float32)[None]
    for S in (1, 2):
        r = O.int16_residual(A, 1, True, S, parts=True)
        assert np.array_equal(r["E"][0], G["E16"])
        assert np.array_equal(r["qE"][0], G["qE16"].astype(np.int64))
        assert r["sE"][0] == 2.0 ** -16
        assert np.array_equal(r["Gm"][0], G["Gm16"])
        assert np.array_equal(r["T"][0], G["T16"].astype(np.float32))
    Z = np.zeros((1, 4, 4), np.float32)
    Z[0, 3, 2] = -0.25
    r = O.int16_residual(Z, 1, True, 2, parts=True)
    assert not r["E"].any() and r["sE"][0] == 0
    assert np.array_equal(r["T"][0], np.eye(4, dtype=np.float32) + Z[0])


def _int8_residual_variant(A32, N, mask, S, swap=None):
    """The INT8 residual written out again with one documented float32
    operation order swapped (``swap``), for the test below: a planted mistake
    that must change the result bits on realistic chunks."""
    f32 = np.float32
    nc, k, _ = A32.shape

    def codes(x):
        amax = np.abs(x).reshape(nc, -1).max(axis=1).astype(f32)
        safe = np.where(amax > 0, amax, f32(1.0)).astype(f32)
        r = (f32(127.0) / safe).astype(f32)
        q = np.clip(np.rint((x * r[:, None, None]).astype(f32)), -127, 127).astype(np.int64)
        q = np.where((amax > 0)[:, None, None], q, 0)
        return q, np.where(amax > 0, (amax / f32(127.0)).astype(f32), f32(0.0)).astype(f32)

    def deq(sa, sb, acc):
        if swap == "deq_order":           # s_a (s_b acc) instead of (s_a s_b) acc
            return (sa[:, None, None] * (sb[:, None, None] * acc.astype(f32)).astype(f32)).astype(f32)
        return ((sa * sb).astype(f32)[:, None, None] * acc.astype(f32)).astype(f32)

    T0 = O.int8_neumann(A32, N, mask)["T"]
    X = (T0 - np.eye(k, dtype=f32)).astype(f32)
    qA, sA = codes(A32)
    qX, sX = codes(X)
    D = deq(sA, sX, qA @ qX)
    if swap == "E_order":                 # A - (X - D) instead of (A - X) + D
        E = (A32 - (X - D).astype(f32)).astype(f32)
    else:
        E = ((A32 - X).astype(f32) + D).astype(f32)
    qE, sE = codes(E)
    qs, ss = qE, sE
    terms = [(ss[:, None, None] * qs.astype(f32)).astype(f32)]
    for _ in range(2, S + 1):
        acc = qs @ qE
        m = np.abs(acc).reshape(nc, -1).max(axis=1)
        mf = m.astype(f32)
        safe = np.where(m > 0, mf, f32(1.0)).astype(f32)
        r = (f32(127.0) / safe).astype(f32)
        q = np.clip(np.rint((acc.astype(f32) * r[:, None, None]).astype(f32)), -127, 127)
        qs = np.where((m > 0)[:, None, None], q.astype(np.int64), 0)
        if swap == "scale_order":         # s_{s-1} (s_E (m / 127)) instead of (s_{s-1} s_E)(m / 127)
            ss_new = (ss * (sE * (mf / f32(127.0)).astype(f32)).astype(f32)).astype(f32)
        else:
            ss_new = ((ss * sE).astype(f32) * (mf / f32(127.0)).astype(f32)).astype(f32)
        ss = np.where(m > 0, ss_new, f32(0.0)).astype(f32)
        terms.append((ss[:, None, None] * qs.astype(f32)).astype(f32))
    if swap == "sum_order":               # sum from s = S down to 1
        terms = terms[::-1]
    Gm = terms[0]
    for t in terms[1:]:
        Gm = (Gm + t).astype(f32)
    qG, sG = codes(Gm)
    D2 = deq(sX, sG, qX @ qG)
    if swap == "T_order":                 # T0 + (Gm + D2) instead of (T0 + Gm) + D2
        return (T0 + (Gm + D2).astype(f32)).astype(f32)
    return ((T0 + Gm).astype(f32) + D2).astype(f32)


def test_int8_residual_operation_order_is_seen():
    """Every float32 operation order that the INT8 residual fixes changes the
    result bits on realistic chunks when swapped, so the bit-exact GPU
    comparison on such chunks pins the order, not only the formula."""
    K, _, beta, g, _ = random_chunks(16, 64, 128, seed=31)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    ref = O.int8_residual(A32, 3, True, 8)
    assert np.array_equal(_int8_residual_variant(A32, 3, True, 8), ref)     # the order as written
    for swap in ("deq_order", "scale_order", "sum_order", "T_order"):
        assert not np.array_equal(_int8_residual_variant(A32, 3, True, 8, swap), ref), swap
    # The order of E = (A - X) + D is the one step the result cannot see: off
    # the band X = 0 and both orders are A + D, and in the band the float32
    # difference of A - (X - D) never moves a code (E is quantised next).
    assert np.array_equal(_int8_residual_variant(A32, 3, True, 8, "E_order"), ref)


def test_int16_codes_and_int64_accumulators():
    k, N = 16, 4
    K, _, beta, g, _ = random_chunks(3, k, 16, seed=14, gate_scale=0.2)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    dist = np.arange(k)[:, None] - np.arange(k)[None, :]
    for mask in (False, True):
        r = O.int16_neumann(A32, N, mask)
        q, acc = r["q"], r["acc"]
        assert q.min() >= -32767 and q.max() <= 32767
        assert np.any(np.abs(q[:, 0]) == 32767)
        for n in range(1, N):
            for c in range(3):
                for i in range(k):
                    for j in range(k):
                        want = sum(int(q[c, n - 1, i, l]) * int(q[c, 0, l, j]) for l in range(k))
                        if mask and dist[i, j] > N:
                            want = 0
                        assert int(acc[c, n, i, j]) == want
                # the code of the largest accumulator is +-32767
                assert np.abs(q[c, n]).max() in (0, 32767)
        if mask:
            assert np.all(q[:, :, dist > N] == 0)


def test_int16_rounding_and_scale_by_hand():
    A = np.zeros((1, 4, 4), np.float32)
    A[0, 1, 0] = 32767.0                 # r = 1 exactly: the codes are rint of the entries
    A[0, 2, 0] = 2.5
    A[0, 2, 1] = -1.5
    A[0, 3, 2] = 1000.5
    r = O.int16_neumann(A, 2, False)
    assert r["q"][0, 0, 1, 0] == 32767
    assert r["q"][0, 0, 2, 0] == 2 and r["q"][0, 0, 2, 1] == -2 and r["q"][0, 0, 3, 2] == 1000
    assert r["scale"][0, 0] == 1.0
    # A^2 by hand: (2,0) += 0, (3,1) = 1000 * -2, (3,0) = 1000 * 2, (2,0) = -2 * 32767
    A2 = np.zeros((4, 4), np.int64)
    A2[2, 0] = -2 * 32767
    A2[3, 0] = 1000 * 2
    A2[3, 1] = 1000 * -2
    assert np.array_equal(r["acc"][0, 1], A2)
    assert r["scale"][0, 1] == 1.0 * 1.0 * (2 * 32767 / 32767.0)
    assert r["q"][0, 1, 2, 0] == -32767 and r["q"][0, 1, 3, 0] == 1000


def test_int16_dequantised_much_closer_than_int8():
    k, N = 64, 3
    K, _, beta, g, _ = random_chunks(6, k, 128, seed=15)
    A32 = O.build_A(K, beta, g).astype(np.float32)
    for mask in (False, True):
        ref = O.invert_neumann(A32.astype(np.float64), N, mask, 0)
        e16 = O.rel_fro(O.int16_neumann(A32, N, mask)["T"], ref)
        e8 = O.rel_fro(O.int8_neumann(A32, N, mask)["T"], ref)
        assert e16 <= 1e-4 and e16 < e8 / 50


def test_int8_dequantised_close_to_float64():
    k, N = 64, 3
    K, _, beta, g, _ = random_chunks(8, k, 128, seed=13)
    A = O.build_A(K, beta, g)
    A32 = A.astype(np.float32)
    for mask in (False, True):
        r = O.int8_neumann(A32, N, mask)
        ref = O.invert_neumann(A32.astype(np.float64), N, mask, 0)
        # each power carries at most half a code step (1/254 of its max) of error
        assert O.rel_fro(r["T"], ref) <= 1e-2


def test_error_table_follows_the_truncation_laws():
    """The reported error table (``oracle/error_table.py``) on a few chunks of
    the B=4, H=16, T=4096 workload: without the mask and residual the error of
    T falls with every added power; the masked series is exact on its band but
    loses the entries below it, so its error is the larger one at S = 0; the
    residual (S = 8) leaves only rounding; W inherits T's error (W = T diag(b) K)."""
    from oracle.error_table import error_table

    res = error_table(n_chunks=6, Ns=(1, 2, 3), Ss=(0, 8))
    err = {(r["N"], r["mask"], r["S"]): r for r in res["rows"]}
    unmasked = [err[(N, 0, 0)]["T_rel_fro"] for N in (1, 2, 3)]
    assert unmasked[0] > unmasked[1] > unmasked[2] > 0
    for N in (1, 2, 3):
        assert err[(N, 1, 0)]["T_rel_fro"] > err[(N, 0, 0)]["T_rel_fro"]
        assert err[(N, 1, 8)]["T_rel_fro"] < 1e-12
        assert err[(N, 0, 8)]["T_rel_fro"] < 1e-12
        r = err[(N, 1, 0)]
        assert 0.5 * r["T_rel_fro"] < r["W_rel_fro"] < 2.0 * r["T_rel_fro"]
        assert r["T_worst_chunk"] >= r["T_rel_fro"] * 0.999
        assert math.isclose(r["T_snr_db"], -20 * math.log10(r["T_rel_fro"]))
    # the masked powers shrink with n on these fast-decaying gates
    amax = res["amax_masked_powers"][3]
    assert amax[0] > amax[1] > amax[2] > 0
    # the quantised series: INT16 stays orders of magnitude closer to the
    # float64 series than INT8; the float64 row repeats the S = 0 error above
    for q in res["quantised"]:
        assert 0 < q["int16_vs_float"] < q["int8_vs_float"] / 30
        assert math.isclose(q["float_rel_fro"], err[(q["N"], q["mask"], 0)]["T_rel_fro"])


def test_series_and_residual_band_laws_on_random_shapes():
    """Property check over random chunk sizes, orders, masks and strictly
    lower-triangular A (entries up to 0.9 in size, so far entries stay large):
    the truncated series equals the exact inverse on sub-diagonals 0..N (and,
    masked, is zero below); with the residual it is exact on sub-diagonals
    0..(S+1)(N+1)-1 and differs on the next one; a sum long enough to cover
    the chunk is the exact inverse."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    @hyp.settings(max_examples=60, deadline=None, derandomize=True)
    @hyp.given(k=st.integers(2, 24), N=st.integers(1, 6), S=st.integers(0, 4),
               mask=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
    def check(k, N, S, mask, seed):
        rng = np.random.default_rng(seed)
        A = np.tril(rng.uniform(-0.9, 0.9, size=(1, k, k)), -1)
        T = O.invert_fwdsub(A)
        dist = np.arange(k)[:, None] - np.arange(k)[None, :]
        scale = max(1.0, float(np.abs(T).max()))
        T0 = O.invert_neumann(A, N, mask, 0)
        assert np.abs(T0 - T)[:, (dist >= 0) & (dist <= N)].max() <= 1e-12 * scale
        if mask:
            assert not T0[:, dist > N].any()
        L = (S + 1) * (N + 1)
        Tr = O.invert_neumann(A, N, mask, S)
        err = np.abs(Tr - T)
        assert err[:, (dist >= 0) & (dist <= min(L, k) - 1)].max() <= 1e-10 * scale ** (S + 2)
        if L >= k:
            assert O.rel_fro(Tr, T) <= 1e-10 * scale ** (S + 2)
        else:
            assert err[:, dist == L].max() > 0          # the first sub-diagonal left out

    check()
