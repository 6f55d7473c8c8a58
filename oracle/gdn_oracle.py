"""Plain float64 CPU oracle for the per-chunk Gated DeltaNet inversion and WY factors.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg, never by the product path.  Independent of
the CUDA library (no shared code, no imports either way).

Sources.  The method is the one of "When Good Enough Is Optimal:
Multiplication-Only Matrix Inversion Approximation for Quantized Gated
DeltaNet" (arXiv 2606.06034), read through its gist.science technical summary
(sections "Énoncé du Problème", "Méthodologie" §1-§3, "Adaptation à la
Quantification", "Études d'Ablation") and its deepcamp.cc abstract page; the
decode step follows the technical summary of "A Persistent-State Dataflow
Accelerator for Memory-Bound Linear Attention Decode on FPGA".  The
pages do not print A's entries nor the Gated DeltaNet recurrence; those come
from the textbook gated delta rule

    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,

whose chunk form (derived in ``chunk_forward``'s docstring) yields the
strictly lower-triangular system (I - A) V~ = ... with
A_ij = -b_i (k_i . k_j) exp(g_i - g_j) for i > j.

Array conventions: a "chunk batch" is an array whose two trailing axes are one
chunk: ``A, T: [nc, k, k]``, ``K, V: [nc, k, d]``, ``beta, g: [nc, k]``.
Use ``to_chunks`` to go from ``[B, H, T, ...]`` to ``[nc, k, ...]``.

Parity pins: every function below is pinned by ``tests/test_oracle_pins.py``
against invariants, closed forms and exact rational brute force; none is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "to_chunks", "from_chunks", "l2_normalize_rows", "chunk_cumsum", "band_mask", "build_A",
    "invert_fwdsub",
    "neumann_powers_sum", "invert_neumann", "invert_newton", "invert_blocked", "residual_matrix",
    "wy",
    "int8_neumann", "int8_residual", "int16_neumann", "int16_residual", "chunk_forward", "token_recurrence", "decode", "rel_fro", "snr_db",
]


# --------------------------------------------------------------------------- #
# layout helpers (no arithmetic of the method)
# --------------------------------------------------------------------------- #
def to_chunks(x: np.ndarray, k: int) -> np.ndarray:
    """``[B, H, T, *rest] -> [B*H*T/k, k, *rest]`` (chunks are contiguous in T)."""
    B, H, T = x.shape[:3]
    return x.reshape(B * H * (T // k), k, *x.shape[3:])


def from_chunks(x: np.ndarray, B: int, H: int) -> np.ndarray:
    """Inverse of ``to_chunks``: ``[nc, k, *rest] -> [B, H, T, *rest]``."""
    nc, k = x.shape[:2]
    return x.reshape(B, H, (nc // (B * H)) * k, *x.shape[2:])


def rel_fro(x: np.ndarray, ref: np.ndarray) -> float:
    """Relative Frobenius error ||x - ref||_F / ||ref||_F, in float64."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm((x - ref).ravel()) / np.linalg.norm(ref.ravel()))


def snr_db(x: np.ndarray, ref: np.ndarray) -> float:
    """Signal-to-noise ratio 10 log10(||ref||^2 / ||x - ref||^2) in dB."""
    err = rel_fro(x, ref)
    return float("inf") if err == 0.0 else float(-20.0 * np.log10(err))


# --------------------------------------------------------------------------- #
# the prologue: key normalisation and chunk-local cumulative gates
# --------------------------------------------------------------------------- #
def l2_normalize_rows(K: np.ndarray) -> np.ndarray:
    """k_i / ||k_i||_2 over the last axis; an all-zero row stays zero.  The
    workloads' keys are unit rows ("K rows N(0,1) then L2-normalised")."""
    K = np.asarray(K, np.float64)
    n = np.sqrt(np.sum(K * K, axis=-1, keepdims=True))
    return np.divide(K, n, out=np.zeros_like(K), where=n > 0)


def chunk_cumsum(loggate: np.ndarray, k: int) -> np.ndarray:
    """Inclusive cumulative sum of the per-token log-gates over the last axis,
    restarted every ``k`` entries (the chunk-local g; g_i includes token i)."""
    x = np.asarray(loggate, np.float64)
    T = x.shape[-1]
    return np.cumsum(x.reshape(*x.shape[:-1], T // k, k), axis=-1).reshape(x.shape)


# --------------------------------------------------------------------------- #
# A, exact inverse, truncated Neumann + mask + residual
# --------------------------------------------------------------------------- #
def band_mask(k: int, N: int) -> np.ndarray:
    """Structural diagonal mask M^(N): M_ij = 1 if i - j <= N else 0.

    "When Good Enough Is Optimal", Méthodologie §2 (masquage diagonal
    structurel): entries farther than the truncation order N below the main
    diagonal are set to zero.
    """
    i = np.arange(k)[:, None]
    j = np.arange(k)[None, :]
    return (i - j <= N).astype(np.float64)


def build_A(K: np.ndarray, beta: np.ndarray, g: np.ndarray) -> np.ndarray:
    """A_ij = -beta_i (k_i . k_j) exp(g_i - g_j) for i > j, else 0 (per chunk).

    The summary's problem statement ("Énoncé du Problème") fixes only that A is
    strictly lower triangular; the entries are those of the gated delta-rule
    chunk system (see ``chunk_forward``).  exp is evaluated only where i > j,
    so a large positive g_i - g_j above the diagonal can never overflow.
    """
    K = np.asarray(K, np.float64)
    beta = np.asarray(beta, np.float64)
    g = np.asarray(g, np.float64)
    k = K.shape[-2]
    G = K @ np.swapaxes(K, -1, -2)                       # k_i . k_j
    lower = np.tril(np.ones((k, k), dtype=bool), -1)     # i > j
    diff = g[..., :, None] - g[..., None, :]             # g_i - g_j
    gate = np.exp(np.where(lower, diff, 0.0))
    A = -beta[..., :, None] * G * gate
    return np.where(lower, A, 0.0)


def invert_fwdsub(A: np.ndarray) -> np.ndarray:
    """Exact T = (I - A)^{-1} by forward substitution (row by row).

    "When Good Enough Is Optimal", Énoncé du Problème: the reference way of
    inverting the unit lower-triangular I - A takes k - 1 sequential steps.
    From (I - A) T = I, row i of T is e_i + sum_{l < i} A_il T_l.
    """
    A = np.asarray(A, np.float64)
    k = A.shape[-1]
    T = np.zeros_like(A)
    for i in range(k):
        T[..., i, i] = 1.0
        if i:
            T[..., i, :] += np.einsum("...l,...lj->...j", A[..., i, :i], T[..., :i, :])
    return T


def neumann_powers_sum(A: np.ndarray, n_max: int) -> np.ndarray:
    """sum_{n=0}^{n_max} A^n with the powers formed by repeated products A^n = A^{n-1} A.

    "When Good Enough Is Optimal", Méthodologie §1: T^(0) = sum_{n=0}^{N} A^n.
    With n_max = k - 1 this is the exact inverse, since A^k = 0 (Lemma 3.1).
    """
    A = np.asarray(A, np.float64)
    k = A.shape[-1]
    eye = np.broadcast_to(np.eye(k), A.shape)
    P = eye.copy()
    acc = eye.copy()
    for _ in range(n_max):
        P = P @ A
        acc = acc + P
    return acc


def residual_matrix(A: np.ndarray, T0: np.ndarray) -> np.ndarray:
    """E = I - (I - A) T^(0).

    "When Good Enough Is Optimal", Méthodologie §3 (correction de résidu
    parallèle): the residual error of the initial approximation.
    """
    A = np.asarray(A, np.float64)
    k = A.shape[-1]
    eye = np.eye(k)
    return eye - (eye - A) @ T0


def invert_blocked(A: np.ndarray, base: int = 16) -> np.ndarray:
    """Exact T = (I - A)^{-1} by 2 x 2 block decomposition, the alternative the
    summary of "When Good Enough Is Optimal" sets against its method (Énoncé
    du Problème: block inversion).  With I - A = [[L00, 0], [-A10, L11]]:

      T = [[T00, 0], [T11 A10 T00, T11]],  T00 = L00^{-1},  T11 = L11^{-1},

    recursively down to ``base`` x ``base`` blocks, which are inverted by
    forward substitution.  ``A: [..., k, k]`` with k = base * 2^m.
    """
    A = np.asarray(A, np.float64)
    k = A.shape[-1]
    if k <= base:
        return invert_fwdsub(A)
    hk = k // 2
    T00 = invert_blocked(A[..., :hk, :hk], base)
    T11 = invert_blocked(A[..., hk:, hk:], base)
    T = np.zeros(A.shape)
    T[..., :hk, :hk] = T00
    T[..., hk:, hk:] = T11
    T[..., hk:, :hk] = T11 @ A[..., hk:, :hk] @ T00
    return T


def invert_neumann(A: np.ndarray, N: int, mask: bool, S: int) -> np.ndarray:
    """Multiplication-only approximate inverse of I - A.

    Steps, in the order of "When Good Enough Is Optimal", Méthodologie:

    1. §1: T^(0) = sum_{n=0}^{N} A^n (N + 1 terms; N = 1 means I + A);
    2. §2: if ``mask``, T^(0) <- M^(N) (.) T^(0) (element-wise), M_ij = [i - j <= N];
    3. §3: if S > 0, E = I - (I - A) T^(0) and T = T^(0) sum_{s=0}^{S} E^s
       (S + 1 terms, literal powers E^s = E^{s-1} E); S = 0 returns T^(0).

    The mask multiplies the truncated sum, as the summary states it; masking
    every power as it is formed gives the same matrix in exact arithmetic.
    """
    if N < 0 or S < 0:
        raise ValueError("N and S must be >= 0")
    A = np.asarray(A, np.float64)
    k = A.shape[-1]
    T0 = neumann_powers_sum(A, N)
    if mask:
        T0 = T0 * band_mask(k, N)
    if S == 0:
        return T0
    E = residual_matrix(A, T0)
    eye = np.broadcast_to(np.eye(k), A.shape)
    Ep = eye.copy()
    acc = eye.copy()
    for _ in range(S):
        Ep = Ep @ E
        acc = acc + Ep
    return T0 @ acc


def invert_newton(A: np.ndarray, N: int, mask: bool, M: int) -> np.ndarray:
    """Sequential residual correction, the comparison point of "When Good Enough
    Is Optimal", Méthodologie §3: the iterative update T^(m+1) = T^(m) +
    T^(m) R^(m) that the method replaces by its parallel sum, with the plain
    reading R^(m) = I - (I - A) T^(m) (the residual of the current iterate).
    T^(0) is the truncated, optionally masked series of ``invert_neumann``;
    ``M`` steps are applied.
    """
    if M < 0:
        raise ValueError("M must be >= 0")
    A = np.asarray(A, np.float64)
    T = invert_neumann(A, N, mask, 0)
    for _ in range(M):
        R = residual_matrix(A, T)
        T = T + T @ R
    return T


def wy(T: np.ndarray, K: np.ndarray, V: np.ndarray, beta: np.ndarray,
       g: np.ndarray | None = None):
    """WY factors W = T diag(beta) K and U = T diag(beta) V.

    With ``g`` given, W is the gated factor W_g = T diag(beta * exp(g)) K that
    the chunk recurrence needs (see ``chunk_forward``); U is unchanged.
    """
    T = np.asarray(T, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    beta = np.asarray(beta, np.float64)
    bw = beta if g is None else beta * np.exp(np.asarray(g, np.float64))
    W = T @ (bw[..., :, None] * K)
    U = T @ (beta[..., :, None] * V)
    return W, U


# --------------------------------------------------------------------------- #
# INT8 quantised truncated Neumann (integer + IEEE float32)
# --------------------------------------------------------------------------- #
def int8_neumann(A32: np.ndarray, N: int, mask: bool) -> dict:
    """INT8 truncated Neumann series with symmetric per-chunk scales.

    "When Good Enough Is Optimal", Adaptation à la Quantification and
    Méthodologie §2: A and each power A^n are held as int8 codes with one
    float32 scale per chunk and power, products accumulate in int32, and the
    structural mask is applied to every power before it is quantised (keeping
    the large lower-left entries out of the codes).  The pages fix neither the
    rounding nor the order of the float32 operations; this oracle fixes them
    (all IEEE float32, round to nearest even, no fused multiply-add):

      1. P_1 = M (.) A (the mask, when on, acts before quantising);
         a = max |P_1| over the chunk;  r = 127 / a;
         q_1 = clamp(rint(P_1 * r), -127, 127);  s_1 = a / 127;
      2. for n = 2..N: acc_n = q_{n-1} q_1 (exact int32), masked;
         m_n = max |acc_n|;  r_n = 127 / float(m_n);
         q_n = clamp(rint(float(acc_n) * r_n), -127, 127);
         s_n = (s_{n-1} * s_1) * (float(m_n) / 127);
      3. a zero maximum gives q = 0 and s = 0 (no division);
      4. T^(0) = I + sum_{n=1}^{N} s_n * float(q_n), accumulated in float32 in
         the order n = 1..N.

    ``A32`` must be float32 ``[nc, k, k]``.  Returns a dict with ``q``
    (int8 ``[nc, N, k, k]``), ``acc`` (int32 ``[nc, N, k, k]``; slot 0 is
    zero, there is no product for n = 1), ``scale`` (float32 ``[nc, N]``) and
    ``T`` (float32 ``[nc, k, k]``).
    """
    if N < 1:
        raise ValueError("the INT8 path needs N >= 1")
    A32 = np.asarray(A32)
    if A32.dtype != np.float32:
        raise TypeError("A32 must be float32")
    nc, k, _ = A32.shape
    f32 = np.float32
    M = band_mask(k, N).astype(bool) if mask else np.ones((k, k), dtype=bool)

    def quantise(x: np.ndarray, xmax: np.ndarray) -> np.ndarray:
        # x float32 [nc,k,k], xmax float32 [nc] (> 0 where used)
        safe = np.where(xmax > 0, xmax, f32(1.0)).astype(f32)
        r = (f32(127.0) / safe).astype(f32)
        y = (x * r[:, None, None]).astype(f32)
        q = np.clip(np.rint(y), -127, 127).astype(np.int8)
        return np.where((xmax > 0)[:, None, None], q, np.int8(0))

    q = np.zeros((nc, N, k, k), np.int8)
    acc = np.zeros((nc, N, k, k), np.int32)
    scale = np.zeros((nc, N), f32)

    A1 = np.where(M, A32, f32(0.0)).astype(f32)              # P_1 = M (.) A
    amax = np.abs(A1).reshape(nc, -1).max(axis=1).astype(f32)
    q1 = quantise(A1, amax)
    q[:, 0] = q1
    scale[:, 0] = np.where(amax > 0, (amax / f32(127.0)).astype(f32), f32(0.0))
    q1_64 = q1.astype(np.int64)
    for n in range(1, N):
        prod = q[:, n - 1].astype(np.int64) @ q1_64        # exact
        prod = np.where(M, prod, 0)
        assert np.abs(prod).max(initial=0) < 2 ** 31
        acc[:, n] = prod.astype(np.int32)
        m = np.abs(prod).reshape(nc, -1).max(axis=1)
        mf = m.astype(f32)                                  # exact: m < 2^24
        q[:, n] = quantise(prod.astype(f32), mf)
        s = ((scale[:, n - 1] * scale[:, 0]).astype(f32)
             * (mf / f32(127.0)).astype(f32)).astype(f32)
        scale[:, n] = np.where(m > 0, s, f32(0.0))

    T = np.broadcast_to(np.eye(k, dtype=f32), (nc, k, k)).copy()
    for n in range(N):
        T = (T + (scale[:, n, None, None] * q[:, n].astype(f32)).astype(f32)).astype(f32)
    return {"q": q, "acc": acc, "scale": scale, "T": T}


def int8_residual(A32: np.ndarray, N: int, mask: bool, S: int, parts: bool = False):
    """INT8 series followed by the parallel residual correction, every product
    an int8 product ("When Good Enough Is Optimal", Adaptation à la
    Quantification: N = 3 compensated by S = 8 residual steps; Méthodologie
    §3 for E and T = T^(0) sum E^s).  The pages fix neither how E is formed
    nor the precision of the last product; this reading keeps every matrix
    product in int8 codes with the rules of ``int8_neumann`` (per-chunk
    symmetric scales, int32 accumulators, IEEE float32 without FMA, round to
    nearest even, zero maxima give zero codes and scales):

      1. T^(0) from ``int8_neumann``; X = T^(0) - I (exact: T^(0)_ii = 1);
      2. codes of the whole A (no mask) and of X: (q_A, s_A), (q_X, s_X);
         E = (A - X) + (s_A * s_X) * float(q_A q_X)   [= I - (I - A) T^(0)];
      3. codes of E: (q_E1, s_E1); for s = 2..S: acc = q_E,s-1 q_E1,
         q_E,s and s_E,s requantised as the powers of A (E is not masked);
         Gm = sum_{s=1}^{S} s_E,s * float(q_E,s), left to right from s = 1;
      4. codes of Gm: (q_G, s_G);
         T = (T^(0) + Gm) + (s_X * s_G) * float(q_X q_G)   [= T^(0) (I + Gm)].

    ``A32`` float32 ``[nc, k, k]``; returns T float32 ``[nc, k, k]``, or with
    ``parts`` a dict that also holds E, its codes and scale (``qE``, ``sE``),
    Gm and its codes and scale (``qG``, ``sG``).
    """
    if S < 1:
        raise ValueError("the residual needs S >= 1")
    f32 = np.float32
    A32 = np.asarray(A32)
    if A32.dtype != np.float32:
        raise TypeError("A32 must be float32")
    nc, k, _ = A32.shape

    def codes(x):
        # (int64 codes, float32 scale per chunk) of a float32 [nc, k, k] array
        amax = np.abs(x).reshape(nc, -1).max(axis=1).astype(f32)
        safe = np.where(amax > 0, amax, f32(1.0)).astype(f32)
        r = (f32(127.0) / safe).astype(f32)
        q = np.clip(np.rint((x * r[:, None, None]).astype(f32)), -127, 127).astype(np.int64)
        q = np.where((amax > 0)[:, None, None], q, 0)
        sc = np.where(amax > 0, (amax / f32(127.0)).astype(f32), f32(0.0)).astype(f32)
        return q, sc

    def deq(sa, sb, acc):
        # (s_a * s_b) * float(acc), float32 (|acc| < 2^24: exact in float32)
        assert np.abs(acc).max(initial=0) < 2 ** 24
        return ((sa * sb).astype(f32)[:, None, None] * acc.astype(f32)).astype(f32)

    T0 = int8_neumann(A32, N, mask)["T"]
    X = (T0 - np.eye(k, dtype=f32)).astype(f32)
    qA, sA = codes(A32)
    qX, sX = codes(X)
    E = ((A32 - X).astype(f32) + deq(sA, sX, qA @ qX)).astype(f32)
    qE, sE = codes(E)
    qs, ss = qE, sE
    Gm = (ss[:, None, None] * qs.astype(f32)).astype(f32)
    for _ in range(2, S + 1):
        acc = qs @ qE
        assert np.abs(acc).max(initial=0) < 2 ** 31
        m = np.abs(acc).reshape(nc, -1).max(axis=1)
        mf = m.astype(f32)
        safe = np.where(m > 0, mf, f32(1.0)).astype(f32)
        r = (f32(127.0) / safe).astype(f32)
        q = np.clip(np.rint((acc.astype(f32) * r[:, None, None]).astype(f32)), -127, 127)
        qs = np.where((m > 0)[:, None, None], q.astype(np.int64), 0)
        ss = np.where(m > 0, ((ss * sE).astype(f32) * (mf / f32(127.0)).astype(f32)).astype(f32),
                      f32(0.0)).astype(f32)
        Gm = (Gm + (ss[:, None, None] * qs.astype(f32)).astype(f32)).astype(f32)
    qG, sG = codes(Gm)
    T = ((T0 + Gm).astype(f32) + deq(sX, sG, qX @ qG)).astype(f32)
    if parts:
        return {"E": E, "qE": qE, "sE": sE, "Gm": Gm, "qG": qG, "sG": sG, "T": T}
    return T


def int16_neumann(A32: np.ndarray, N: int, mask: bool) -> dict:
    """INT16 truncated Neumann series with symmetric per-chunk scales.

    "When Good Enough Is Optimal", Adaptation à la Quantification: the INT16
    operating point beside INT8.  Same steps as ``int8_neumann`` with codes in
    [-32767, 32767]; products of two code matrices reach 2^36, beyond float32's
    exact integers, so the accumulators are int64 and every scale operation is
    IEEE binary64 (round to nearest even, no fused multiply-add):

      1. P_1 = M (.) A;  a = max |P_1|;  r = 32767 / double(a);
         q_1 = clamp(rint(double(P_1) * r), -32767, 32767);  s_1 = double(a) / 32767;
      2. for n = 2..N: acc_n = q_{n-1} q_1 (exact int64), masked;
         m_n = max |acc_n|;  r_n = 32767 / double(m_n);
         q_n = clamp(rint(double(acc_n) * r_n), -32767, 32767);
         s_n = (s_{n-1} * s_1) * (double(m_n) / 32767);
      3. a zero maximum gives q = 0 and s = 0;
      4. T^(0) = I + sum_{n=1}^{N} s_n * double(q_n), summed in binary64 in the
         order n = 1..N, then rounded once to float32.

    ``A32`` float32 ``[nc, k, k]``.  Returns ``q`` (int16 ``[nc, N, k, k]``),
    ``acc`` (int64, slot 0 zero), ``scale`` (float64 ``[nc, N]``) and ``T``
    (float32).
    """
    if N < 1:
        raise ValueError("the INT16 path needs N >= 1")
    A32 = np.asarray(A32)
    if A32.dtype != np.float32:
        raise TypeError("A32 must be float32")
    nc, k, _ = A32.shape
    M = band_mask(k, N).astype(bool) if mask else np.ones((k, k), dtype=bool)

    def quantise(x: np.ndarray, xmax: np.ndarray) -> np.ndarray:
        # x float64 [nc,k,k], xmax float64 [nc] (> 0 where used)
        safe = np.where(xmax > 0, xmax, 1.0)
        r = 32767.0 / safe
        q = np.clip(np.rint(x * r[:, None, None]), -32767, 32767).astype(np.int16)
        return np.where((xmax > 0)[:, None, None], q, np.int16(0))

    q = np.zeros((nc, N, k, k), np.int16)
    acc = np.zeros((nc, N, k, k), np.int64)
    scale = np.zeros((nc, N), np.float64)
    A1 = np.where(M, A32, np.float32(0.0)).astype(np.float64)   # P_1 = M (.) A
    amax = np.abs(A1).reshape(nc, -1).max(axis=1)
    q[:, 0] = quantise(A1, amax)
    scale[:, 0] = np.where(amax > 0, amax / 32767.0, 0.0)
    q1 = q[:, 0].astype(np.int64)
    for n in range(1, N):
        prod = np.where(M, q[:, n - 1].astype(np.int64) @ q1, 0)     # exact
        acc[:, n] = prod
        m = np.abs(prod).reshape(nc, -1).max(axis=1)
        mf = m.astype(np.float64)                                   # exact: m < 2^53
        q[:, n] = quantise(prod.astype(np.float64), mf)
        scale[:, n] = np.where(m > 0, (scale[:, n - 1] * scale[:, 0]) * (mf / 32767.0), 0.0)
    T = np.broadcast_to(np.eye(k), (nc, k, k)).copy()
    for n in range(N):
        T = T + scale[:, n, None, None] * q[:, n].astype(np.float64)
    return {"q": q, "acc": acc, "scale": scale, "T": T.astype(np.float32)}


def int16_residual(A32: np.ndarray, N: int, mask: bool, S: int, parts: bool = False):
    """INT16 series followed by the parallel residual correction, every
    product an int16 code product ("When Good Enough Is Optimal", Adaptation
    à la Quantification: the INT16 operating point with N = 3 and S = 8;
    Méthodologie §3 for E and T = T^(0) sum E^s).  The steps of
    ``int8_residual`` under the rules of ``int16_neumann``: codes in
    [-32767, 32767], int64 accumulators (exact), every scale and sum in IEEE
    binary64, zero maxima give zero codes and scales, and T rounded once to
    float32 at the end:

      1. T^(0) = I + sum_n s_n q_n in binary64 (``int16_neumann``'s sum before
         its rounding); X = T^(0) - I;
      2. codes of the whole A (no mask) and of X: (q_A, s_A), (q_X, s_X);
         E = (A - X) + (s_A * s_X) * double(q_A q_X);
      3. codes of E: (q_E1, s_E1); for s = 2..S: acc = q_E,s-1 q_E1,
         m = max |acc|, q_E,s = clamp(rint(double(acc) * (32767 / m))),
         s_E,s = (s_E,s-1 * s_E1) * (m / 32767) (E is not masked);
         Gm = sum_{s=1}^{S} s_E,s * double(q_E,s), left to right;
      4. codes of Gm: (q_G, s_G);
         T = (T^(0) + Gm) + (s_X * s_G) * double(q_X q_G), then float32.

    ``A32`` float32 ``[nc, k, k]``; returns T float32 ``[nc, k, k]``, or with
    ``parts`` a dict that also holds E, its codes and scale (``qE``, ``sE``),
    Gm and its codes and scale (``qG``, ``sG``), all binary64 or int64.
    """
    if S < 1:
        raise ValueError("the residual needs S >= 1")
    A32 = np.asarray(A32)
    if A32.dtype != np.float32:
        raise TypeError("A32 must be float32")
    nc, k, _ = A32.shape

    def codes(x):
        # (int64 codes, binary64 scale per chunk) of a binary64 [nc, k, k] array
        amax = np.abs(x).reshape(nc, -1).max(axis=1)
        safe = np.where(amax > 0, amax, 1.0)
        q = np.clip(np.rint(x * (32767.0 / safe)[:, None, None]), -32767, 32767).astype(np.int64)
        q = np.where((amax > 0)[:, None, None], q, 0)
        return q, np.where(amax > 0, amax / 32767.0, 0.0)

    def deq(sa, sb, acc):
        # (s_a * s_b) * double(acc); |acc| <= k 32767^2 < 2^53, exact in binary64
        assert np.abs(acc).max(initial=0) < 2 ** 53
        return (sa * sb)[:, None, None] * acc.astype(np.float64)

    r16 = int16_neumann(A32, N, mask)
    T0 = np.broadcast_to(np.eye(k), (nc, k, k)).copy()
    for n in range(N):
        T0 = T0 + r16["scale"][:, n, None, None] * r16["q"][:, n].astype(np.float64)
    X = T0 - np.eye(k)
    A = A32.astype(np.float64)
    qA, sA = codes(A)
    qX, sX = codes(X)
    E = (A - X) + deq(sA, sX, qA @ qX)
    qE, sE = codes(E)
    qs, ss = qE, sE
    Gm = ss[:, None, None] * qs.astype(np.float64)
    for _ in range(2, S + 1):
        acc = qs @ qE
        m = np.abs(acc).reshape(nc, -1).max(axis=1)
        mf = m.astype(np.float64)
        safe = np.where(m > 0, mf, 1.0)
        q = np.clip(np.rint(acc.astype(np.float64) * (32767.0 / safe)[:, None, None]),
                    -32767, 32767)
        qs = np.where((m > 0)[:, None, None], q.astype(np.int64), 0)
        ss = np.where(m > 0, (ss * sE) * (mf / 32767.0), 0.0)
        Gm = Gm + ss[:, None, None] * qs.astype(np.float64)
    qG, sG = codes(Gm)
    T = ((T0 + Gm) + deq(sX, sG, qX @ qG)).astype(np.float32)
    if parts:
        return {"E": E, "qE": qE, "sE": sE, "Gm": Gm, "qG": qG, "sG": sG, "T": T}
    return T


# --------------------------------------------------------------------------- #
# full chunk-wise forward and the token recurrence it must equal
# --------------------------------------------------------------------------- #
def chunk_forward(Q, K, V, beta, g, T, S0=None):
    """Chunk-wise Gated DeltaNet forward from per-chunk inverses ``T``.

    The pages split the sequence into chunks to expose parallelism inside the
    sequence ("Énoncé du Problème") but print no equations; this is the chunk
    form of the gated delta rule, derived here.  With v~_t = b_t (v_t - a_t
    S_{t-1} k_t), the recurrence reads S_t = a_t S_{t-1} + v~_t k_t^T.  Inside a
    chunk with chunk-local cumulative log-gates g (g_i includes token i's own
    gate), gamma_i = exp(g_i) and start state S0 (d_v x d_k):

      (I - A) V~ = diag(b) V - diag(b gamma) K S0^T     =>  V~ = U - W_g S0^T,
      O   = diag(gamma) Q S0^T + (Q K^T (.) Gamma (.) L) V~,
      S'  = gamma_last S0 + V~^T diag(exp(g_last - g)) K,

    with U = T diag(b) V, W_g = T diag(b gamma) K, Gamma_ij = exp(g_i - g_j)
    and L the lower triangle including the diagonal.

    Arguments are ``[BH, n, k, *]`` arrays (heads flattened, chunks in order):
    ``Q, K, V: [BH, n, k, d]``, ``beta, g: [BH, n, k]``, ``T: [BH, n, k, k]``;
    ``S0: [BH, d_v, d_k]`` or None (zero).  Returns ``(O [BH, n, k, d_v],
    S_final [BH, d_v, d_k])``, float64.
    """
    Q, K, V, beta, g, T = (np.asarray(x, np.float64) for x in (Q, K, V, beta, g, T))
    BH, n, k, dk = K.shape
    dv = V.shape[-1]
    S = np.zeros((BH, dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.zeros((BH, n, k, dv))
    L = np.tril(np.ones((k, k), dtype=bool))
    for c in range(n):
        q, kk, v, b, gc, Tc = Q[:, c], K[:, c], V[:, c], beta[:, c], g[:, c], T[:, c]
        gam = np.exp(gc)                                            # [BH,k]
        U = Tc @ (b[..., None] * v)
        Wg = Tc @ ((b * gam)[..., None] * kk)
        Vt = U - Wg @ np.swapaxes(S, -1, -2)                        # [BH,k,dv]
        diff = gc[:, :, None] - gc[:, None, :]
        Gam = np.exp(np.where(L, diff, 0.0)) * L
        attn = (q @ np.swapaxes(kk, -1, -2)) * Gam
        O[:, c] = gam[..., None] * (q @ np.swapaxes(S, -1, -2)) + attn @ Vt
        decay = np.exp(gc[:, -1:] - gc)                             # [BH,k]
        S = gam[:, -1, None, None] * S + np.swapaxes(Vt, -1, -2) @ (decay[..., None] * kk)
    return O, S


def token_recurrence(Q, K, V, beta, loggate, S0=None):
    """Token-by-token gated delta rule, the definition the chunk form must equal.

    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T and o_t = S_t q_t with
    a_t = exp(loggate_t); S is d_v x d_k.  Arguments ``[BH, T, d]`` /
    ``[BH, T]``; returns ``(O [BH, T, d_v], S_final [BH, d_v, d_k])``.
    """
    Q, K, V, beta, lg = (np.asarray(x, np.float64) for x in (Q, K, V, beta, loggate))
    BH, T, dk = K.shape
    dv = V.shape[-1]
    S = np.zeros((BH, dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.zeros((BH, T, dv))
    eye = np.eye(dk)
    for t in range(T):
        kt, vt, qt, bt = K[:, t], V[:, t], Q[:, t], beta[:, t]
        at = np.exp(lg[:, t])
        H = eye - bt[:, None, None] * kt[:, :, None] * kt[:, None, :]
        S = at[:, None, None] * (S @ H) + bt[:, None, None] * vt[:, :, None] * kt[:, None, :]
        O[:, t] = np.einsum("bij,bj->bi", S, qt)
    return O, S


# --------------------------------------------------------------------------- #
# decode: the recurrence advanced token by token from a carried state
# --------------------------------------------------------------------------- #
def decode(Q, K, V, beta, loggate, S0):
    """Decode steps of the gated delta rule with grouped query/key heads.

    "A Persistent-State Dataflow Accelerator for Memory-Bound Linear Attention
    Decode on FPGA" (its technical summary, §1 and §2): per generated token
    the whole d_v x d_k state of every value head is updated once, and pairs
    of value heads share one query and one key vector (grouped value heads).
    This is the plain definition, one token at a time:

      S <- a_t S (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S q_t,
      a_t = exp(loggate_t),

    where value head h reads query/key head h // (Hv / Hk).  The summary's
    two-pass rewrite of the step is the kernel's business, not the oracle's.

    ``Q, K: [B, Hk, n, d_k]``, ``V: [B, Hv, n, d_v]``, ``beta, loggate:
    [B, Hv, n]``, ``S0: [B, Hv, d_v, d_k]``.  Returns ``(O [B, Hv, n, d_v],
    S [B, Hv, d_v, d_k])`` in float64.
    """
    Q, K, V, beta, lg, S = (np.array(x, np.float64) for x in (Q, K, V, beta, loggate, S0))
    B, Hk, n, dk = K.shape
    Hv = V.shape[1]
    G = Hv // Hk
    O = np.zeros(V.shape)
    eye = np.eye(dk)
    for b in range(B):
        for h in range(Hv):
            Sh = S[b, h]
            for t in range(n):
                k, q, v = K[b, h // G, t], Q[b, h // G, t], V[b, h, t]
                bt, at = beta[b, h, t], math.exp(lg[b, h, t])
                Sh = at * Sh @ (eye - bt * np.outer(k, k)) + bt * np.outer(v, k)
                O[b, h, t] = Sh @ q
            S[b, h] = Sh
    return O, S
