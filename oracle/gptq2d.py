"""GPTQ-2D oracle: a plain, slow, fp64 CPU restatement of two-sided GPTQ rounding.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` may import or call this module; it shares no code with
the CUDA library.

Source, cited by page title and section:

  [D]  "GPTQ-2D：把一个"四次方"难题压回"三次方"的故事" (digi.intozgc.com summary of the
       GPTQ-2D paper): section "两边都被'牵连'" (the two-sided metric ||A(Z - X)B||^2 and its
       vectorized, Kronecker-metric form); "反对角线上的秘密" (an error at (i, j) reaches only
       (p >= i, q >= j); cells of one anti-diagonal are independent; Theorem 1, any order that
       respects that dependence gives the same result; the dense anti-diagonal update,
       Algorithm 2); "GPTQ-2D 的真正巧思" (the buffered row / column push, Algorithm 3, and
       Theorem 2, its equivalence with Algorithm 2, with the invariant C = L E); "把零散更新拼成
       大块矩阵乘法" (groups of w anti-diagonals with two band updates after each group);
       "存储也要讲究" (the skewed layout: one row per anti-diagonal).

The page describes the algorithms in words only.  Readings (the plainest ones the text supports):

  * Z is an integer matrix and rounding is to the nearest integer, ties to even (the page speaks
    of rounding to integers; a uniform grid is the same problem after scaling X).
  * The metric factors are given as G_A = A^T A (m x m) and G_B = B B^T (n x n), both positive
    definite; ||A E B||_F^2 = tr(E^T G_A E G_B).
  * The one-dimensional algorithm is GPTQ's Cholesky form: with R upper triangular and
    R^T R = M^{-1} for the metric M, position v is rounded, its scaled residual
    η_v = (y_v - round(y_v)) / R_vv is recorded, and every later position k receives
    y_k -= η_v R_vk.  On the row-major vectorization vec(E)[i n + j] = E[i, j] the metric is
    M = G_A ⊗ G_B and its factor is R = R_A ⊗ R_B (R_A^T R_A = G_A^{-1}, R_B^T R_B = G_B^{-1}), so
    the feedback from (i, j) to (p, q) is R_A[i, p] R_B[j, q] / (R_A[i, i] R_B[j, j]): the
    "row-direction" and "column-direction" feedback matrices, non-zero only for p >= i, q >= j.
  * The buffer C of Algorithm 3 holds, per column j, the errors pushed down through R_A:
    C[p, j] = sum over processed i <= p of η[i, j] R_A[i, p] (the page's C = L E).  Rounding (i, j)
    (a) folds η[i, j] R_A[i, i:] into C[i:, j], (b) pushes η[i, j] R_A[i, p] R_B[j, j] down to the
    later cells (p > i) of column j, and (c) pushes R_B[j, q] C[i, j] along row i to the cells
    q > j.  Together (b) and (c) give every cell exactly the sum of Algorithm 2's rectangle
    updates, each cell costing O(m + n).
  * The lazy form processes groups of w consecutive anti-diagonals; inside a group (b) and (c)
    reach only cells of the group, and after the group the same two pushes are applied at once to
    every later cell (the page's two band products; (a) already completed C below the group).

Every function is pinned by tests/test_oracle_gptq2d.py (equalities between the algorithms,
Theorem 1 over random valid orders, the one-sided special case against the pinned GPTQ oracle,
the loss identity, diagonal metrics, brute force on tiny cases).
"""
from __future__ import annotations

import numpy as np


def factor_upper_inverse(G) -> np.ndarray:
    """Upper-triangular R with R^T R = G^{-1} (G positive definite)."""
    G = np.asarray(G, np.float64)
    L = np.linalg.cholesky(np.linalg.inv(G))  # L L^T = G^{-1}
    return L.T.copy()


def loss2d(X, Z, GA, GB) -> float:
    """||A (Z - X) B||_F^2 = tr(E^T G_A E G_B) with E = Z - X ([D] the two-sided metric)."""
    E = np.asarray(Z, np.float64) - np.asarray(X, np.float64)
    return float(np.trace(E.T @ np.asarray(GA, np.float64) @ E @ np.asarray(GB, np.float64)))


def gptq2d_vectorized(X, GA, GB):
    """The definition: one-dimensional GPTQ on the row-major vectorization with the Kronecker
    metric M = G_A ⊗ G_B ([D] "two-sided" section), O(m^2 n^2).  Returns (Z, eta), both [m, n]."""
    X = np.asarray(X, np.float64)
    m, n = X.shape
    M = np.kron(np.asarray(GA, np.float64), np.asarray(GB, np.float64))
    R = factor_upper_inverse(M)
    y = X.reshape(-1).copy()
    N = m * n
    z = np.zeros(N)
    eta = np.zeros(N)
    for v in range(N):
        z[v] = np.rint(y[v])
        eta[v] = (y[v] - z[v]) / R[v, v]
        y[v + 1:] -= eta[v] * R[v, v + 1:]
    return z.reshape(m, n), eta.reshape(m, n)


def _round_cell(Y, RA, RB, i, j):
    z = np.rint(Y[i, j])
    return z, (Y[i, j] - z) / (RA[i, i] * RB[j, j])


def gptq2d_wavefront(X, GA, GB):
    """Algorithm 2 of [D]: anti-diagonals s = 0 .. m + n - 2 in order; every cell of one
    anti-diagonal is rounded from the current Y, then each sends its error to its whole lower-right
    rectangle Y[i:, j:] -= η R_A[i, i:] ⊗ R_B[j, j:] (no cell of the same anti-diagonal lies in it).
    Returns (Z, eta)."""
    Y = np.array(X, np.float64, copy=True)
    m, n = Y.shape
    RA, RB = factor_upper_inverse(GA), factor_upper_inverse(GB)
    Z = np.zeros((m, n))
    eta = np.zeros((m, n))
    for s in range(m + n - 1):
        cells = [(i, s - i) for i in range(max(0, s - n + 1), min(s, m - 1) + 1)]
        for i, j in cells:
            Z[i, j], eta[i, j] = _round_cell(Y, RA, RB, i, j)
        for i, j in cells:
            upd = eta[i, j] * np.outer(RA[i, i:], RB[j, j:])
            upd[0, 0] = 0.0  # the cell itself is already rounded
            Y[i:, j:] -= upd
    return Z, eta


def antidiagonal_order(m: int, n: int):
    """Cells by anti-diagonal s = i + j, rows ascending inside one anti-diagonal."""
    return [(i, s - i) for s in range(m + n - 1)
            for i in range(max(0, s - n + 1), min(s, m - 1) + 1)]


def is_valid_order(order, m: int, n: int) -> bool:
    """True if every cell comes after all cells (i, j) with i <= p, j <= q ([D] Theorem 1)."""
    if sorted(order) != [(i, j) for i in range(m) for j in range(n)]:
        return False
    pos = {c: k for k, c in enumerate(order)}
    return all((i == 0 or pos[(i - 1, j)] < pos[(i, j)]) and
               (j == 0 or pos[(i, j - 1)] < pos[(i, j)]) for i in range(m) for j in range(n))


def gptq2d_buffered(X, GA, GB, order=None):
    """Algorithm 3 of [D] (GPTQ-2D): cells in `order` (any valid order, default anti-diagonals);
    rounding (i, j) folds its error into the buffer C down its column, pushes it down the rest of
    its column, and pushes the buffered C[i, j] along the rest of its row.  O(mn (m + n)).
    Returns (Z, eta, C)."""
    Y = np.array(X, np.float64, copy=True)
    m, n = Y.shape
    RA, RB = factor_upper_inverse(GA), factor_upper_inverse(GB)
    order = antidiagonal_order(m, n) if order is None else list(order)
    if not is_valid_order(order, m, n):
        raise ValueError("order does not respect the dependence (i <= p and j <= q)")
    Z = np.zeros((m, n))
    eta = np.zeros((m, n))
    C = np.zeros((m, n))
    for i, j in order:
        Z[i, j], eta[i, j] = _round_cell(Y, RA, RB, i, j)
        C[i:, j] += eta[i, j] * RA[i, i:]                        # (a) fold into the buffer
        Y[i + 1:, j] -= eta[i, j] * RA[i, i + 1:] * RB[j, j]     # (b) down the column
        Y[i, j + 1:] -= C[i, j] * RB[j, j + 1:]                  # (c) along the row
    return Z, eta, C


def gptq2d_lazy(X, GA, GB, w: int):
    """Lazy form of [D]: groups of w consecutive anti-diagonals.  Inside a group the cells are
    rounded in anti-diagonal order with the buffered pushes (b), (c) restricted to cells of the
    group; after the group, the deferred parts of (b) and (c) reach every later cell at once (the
    two band products).  Returns (Z, eta)."""
    if w < 1:
        raise ValueError("w >= 1")
    Y = np.array(X, np.float64, copy=True)
    m, n = Y.shape
    RA, RB = factor_upper_inverse(GA), factor_upper_inverse(GB)
    Z = np.zeros((m, n))
    eta = np.zeros((m, n))
    C = np.zeros((m, n))
    smax = m + n - 1
    for s0 in range(0, smax, w):
        s1 = min(smax, s0 + w)          # the group: anti-diagonals s0 .. s1 - 1
        cells = [c for c in antidiagonal_order(m, n) if s0 <= c[0] + c[1] < s1]
        for i, j in cells:
            Z[i, j], eta[i, j] = _round_cell(Y, RA, RB, i, j)
            C[i:, j] += eta[i, j] * RA[i, i:]
            for p in range(i + 1, m):                 # (b) inside the group
                if p + j < s1:
                    Y[p, j] -= eta[i, j] * RA[i, p] * RB[j, j]
            for q in range(j + 1, n):                 # (c) inside the group
                if i + q < s1:
                    Y[i, q] -= C[i, j] * RB[j, q]
        # band products: the deferred parts of (b) and (c) for every cell beyond the group
        for i, j in cells:
            for p in range(i + 1, m):
                if p + j >= s1:
                    Y[p, j] -= eta[i, j] * RA[i, p] * RB[j, j]
            for q in range(j + 1, n):
                if i + q >= s1:
                    Y[i, q] -= C[i, j] * RB[j, q]
    return Z, eta


def gptq2d_replay(X, GA, GB, other_Z, band: float = 1e-3):
    """Check another implementation's rounding against the buffered recursion, cell by cell in
    anti-diagonal order, following the other's decisions.  A differing integer is accepted iff it
    is adjacent to this recursion's and the pre-round value lies within `band` of the rounding
    boundary between the two (the decision is taken in another precision); anything else is a
    violation.  Returns dict(n, identical, in_band, violations, eta) with the scaled residuals
    of the followed decisions."""
    Y = np.array(X, np.float64, copy=True)
    m, n = Y.shape
    other = np.asarray(other_Z, np.float64)
    RA, RB = factor_upper_inverse(GA), factor_upper_inverse(GB)
    eta = np.zeros((m, n))
    C = np.zeros((m, n))
    identical = in_band = violations = 0
    for i, j in antidiagonal_order(m, n):
        z_o = np.rint(Y[i, j])
        z_g = other[i, j]
        if z_o == z_g:
            identical += 1
        elif abs(z_o - z_g) == 1 and abs(Y[i, j] - (min(z_o, z_g) + 0.5)) <= band:
            in_band += 1
        else:
            violations += 1
        eta[i, j] = (Y[i, j] - z_g) / (RA[i, i] * RB[j, j])
        C[i:, j] += eta[i, j] * RA[i, i:]
        Y[i + 1:, j] -= eta[i, j] * RA[i, i + 1:] * RB[j, j]
        Y[i, j + 1:] -= C[i, j] * RB[j, j + 1:]
    return dict(n=m * n, identical=identical, in_band=in_band, violations=violations, eta=eta)


def to_skewed(X, fill=0.0):
    """The skewed layout of [D] "存储也要讲究": S[s, j] = X[s - j, j], one row per anti-diagonal
    s = i + j (shape [m + n - 1, n]); a column of X is a vertical run, a row of X a diagonal of
    stride n + 1; the n (n - 1) other entries are padding."""
    X = np.asarray(X)
    m, n = X.shape
    S = np.full((m + n - 1, n), fill, dtype=X.dtype)
    for i in range(m):
        for j in range(n):
            S[i + j, j] = X[i, j]
    return S


def from_skewed(S, m: int, n: int):
    """Inverse of `to_skewed`."""
    S = np.asarray(S)
    X = np.empty((m, n), dtype=S.dtype)
    for i in range(m):
        for j in range(n):
            X[i, j] = S[i + j, j]
    return X
