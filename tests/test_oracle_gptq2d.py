"""Pins of the GPTQ-2D oracle (two-sided rounding, "GPTQ-2D：把一个'四次方'难题压回'三次方'的
故事"): its algorithms against one another and against facts fixed outside this module (the pinned
one-sided GPTQ oracle, a closed-form loss identity, diagonal metrics, brute force)."""
import itertools

import numpy as np
import pytest

from oracle import gptq2d as D
from oracle import gptq_oracle as O


def _pd(k, seed, cond=30.0):
    """A seeded positive-definite k x k matrix with a controlled spread of eigenvalues."""
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.normal(size=(k, k)))
    ev = np.geomspace(1.0, 1.0 / cond, k)
    return (Q * ev) @ Q.T


def _problem(m, n, seed, scale=3.0):
    rng = np.random.default_rng(seed)
    return rng.normal(0, scale, (m, n)), _pd(m, seed + 1), _pd(n, seed + 2)


@pytest.mark.parametrize("m,n,seed", [(3, 4, 1), (5, 5, 2), (6, 3, 3), (1, 7, 4), (7, 1, 5)])
def test_algorithms_agree(m, n, seed):
    """Theorem 2 of the page and the vectorized definition: the dense anti-diagonal update, the
    buffered row / column push and every lazy group width give the same rounding as
    one-dimensional GPTQ on the Kronecker metric."""
    X, GA, GB = _problem(m, n, seed)
    Zv, Ev = D.gptq2d_vectorized(X, GA, GB)
    Zw, Ew = D.gptq2d_wavefront(X, GA, GB)
    Zb, Eb, _ = D.gptq2d_buffered(X, GA, GB)
    assert np.array_equal(Zv, Zw) and np.array_equal(Zv, Zb)
    assert np.allclose(Ev, Ew, atol=1e-10) and np.allclose(Ev, Eb, atol=1e-10)
    for w in (1, 2, 3, 5, m + n):
        Zl, El = D.gptq2d_lazy(X, GA, GB, w)
        assert np.array_equal(Zv, Zl), w
        assert np.allclose(Ev, El, atol=1e-10), w


def test_order_independence_theorem1():
    """Theorem 1: every order that rounds (i, j) after all (i' <= i, j' <= j) gives the same
    result -- row by row, column by column, anti-diagonals, and random valid orders."""
    m, n = 5, 6
    X, GA, GB = _problem(m, n, 7)
    ref, _, _ = D.gptq2d_buffered(X, GA, GB)
    orders = [[(i, j) for i in range(m) for j in range(n)],
              [(i, j) for j in range(n) for i in range(m)]]
    rng = np.random.default_rng(8)
    for _ in range(5):
        # a random linear extension of the grid order: repeatedly take a random ready cell
        done, order = set(), []
        while len(order) < m * n:
            ready = [(i, j) for i in range(m) for j in range(n) if (i, j) not in done and
                     (i == 0 or (i - 1, j) in done) and (j == 0 or (i, j - 1) in done)]
            c = ready[rng.integers(len(ready))]
            done.add(c)
            order.append(c)
        orders.append(order)
    for order in orders:
        assert D.is_valid_order(order, m, n)
        Z, _, _ = D.gptq2d_buffered(X, GA, GB, order=order)
        assert np.array_equal(Z, ref)
    with pytest.raises(ValueError):
        D.gptq2d_buffered(X, GA, GB, order=[(0, 1), (0, 0)] + orders[0][2:])


def test_buffer_invariant():
    """The page's invariant C = L E: after the run, column j of C is R_A^T applied to column j of
    the scaled errors (C[p, j] = sum_{i <= p} η[i, j] R_A[i, p])."""
    X, GA, GB = _problem(4, 5, 9)
    _, eta, C = D.gptq2d_buffered(X, GA, GB)
    RA = D.factor_upper_inverse(GA)
    assert np.allclose(C, RA.T @ eta, atol=1e-12)


def test_one_sided_special_case():
    """With G_B = I the columns are independent one-sided problems with metric G_A: the result is
    the pinned one-sided GPTQ oracle (explicit inverse downdates) run on X^T with H = G_A, on an
    integer grid (Δ = 1, zero point 128, 8-bit codes)."""
    m, n = 6, 5
    X, GA, _ = _problem(m, n, 10)
    Z, _ = D.gptq2d_vectorized(X, GA, np.eye(n))
    Xt = X.T.copy()
    scale = np.ones((n, 1), np.float32)
    zero = np.full((n, 1), 128, np.int32)
    codes, Q, _, _ = O.gptq_explicit(Xt, np.linalg.inv(GA), scale, zero, np.zeros(m, int), 8)
    assert np.array_equal(Z, (codes - 128).T)
    assert np.array_equal(Z, Q.T)
    # and symmetrically with G_A = I (rows independent, metric G_B on each row)
    Z2, _ = D.gptq2d_vectorized(X, np.eye(m), GB := _pd(n, 11))
    scale2 = np.ones((m, 1), np.float32)
    zero2 = np.full((m, 1), 128, np.int32)
    codes2, _, _, _ = O.gptq_explicit(X, np.linalg.inv(GB), scale2, zero2, np.zeros(n, int), 8)
    assert np.array_equal(Z2, codes2 - 128)


def test_diagonal_metrics_are_round_to_nearest():
    """Diagonal G_A and G_B make every feedback term zero: Z = rint(X)."""
    rng = np.random.default_rng(12)
    X = rng.normal(0, 4, (4, 6))
    GA = np.diag(rng.uniform(0.5, 2, 4))
    GB = np.diag(rng.uniform(0.5, 2, 6))
    for Z in (D.gptq2d_vectorized(X, GA, GB)[0], D.gptq2d_buffered(X, GA, GB)[0],
              D.gptq2d_lazy(X, GA, GB, 3)[0]):
        assert np.array_equal(Z, np.rint(X))


def test_loss_identity():
    """||A (Z - X) B||^2 equals the sum of the squared scaled residuals η² (the Cholesky form
    makes the error R^T η with R M R^T = I); A and B are explicit random factors here."""
    rng = np.random.default_rng(13)
    m, n = 5, 4
    A = rng.normal(size=(7, m))
    B = rng.normal(size=(n, 6))
    X = rng.normal(0, 2, (m, n))
    Z, eta, _ = D.gptq2d_buffered(X, A.T @ A, B @ B.T)
    direct = float(np.sum((A @ (Z - X) @ B) ** 2))
    assert np.isclose(direct, float(np.sum(eta ** 2)), rtol=1e-9)
    assert np.isclose(D.loss2d(X, Z, A.T @ A, B @ B.T), direct, rtol=1e-12)


def test_brute_force_tiny():
    """On 2 x 2 problems the exhaustive search over integer matrices near X bounds the greedy
    result from below; on 1 x 1 the greedy result is the optimum (plain rounding)."""
    rng = np.random.default_rng(14)
    for trial in range(10):
        X, GA, GB = _problem(2, 2, 100 + trial, scale=1.5)
        Z, _, _ = D.gptq2d_buffered(X, GA, GB)
        base = np.floor(X)
        best = min(D.loss2d(X, base + np.array(d).reshape(2, 2), GA, GB)
                   for d in itertools.product((-1, 0, 1, 2), repeat=4))
        assert D.loss2d(X, Z, GA, GB) >= best - 1e-12
    x = np.array([[0.37]])
    Z1, _ = D.gptq2d_vectorized(x, np.array([[2.0]]), np.array([[0.5]]))
    assert Z1[0, 0] == 0.0


def test_last_cell_is_conditionally_optimal():
    """The last cell's rounding is the best choice for it given all the others (the greedy step
    is exact for the final coordinate)."""
    X, GA, GB = _problem(4, 4, 15)
    Z, _, _ = D.gptq2d_buffered(X, GA, GB)
    base = D.loss2d(X, Z, GA, GB)
    for dz in (-1.0, 1.0):
        Z2 = Z.copy()
        Z2[-1, -1] += dz
        assert D.loss2d(X, Z2, GA, GB) >= base - 1e-12


def test_skewed_layout():
    """One row per anti-diagonal: a column of X is a vertical run, a row of X a diagonal of stride
    n + 1, the padding is n (n - 1) entries, and the layout round-trips."""
    m, n = 4, 6
    X = np.arange(1, m * n + 1, dtype=float).reshape(m, n)
    S = D.to_skewed(X)
    assert S.shape == (m + n - 1, n)
    assert np.count_nonzero(S == 0) == n * (n - 1)
    for j in range(n):
        assert np.array_equal(S[j:j + m, j], X[:, j])
    flat = S.reshape(-1)
    for i in range(m):
        assert np.array_equal(flat[i * n::n + 1][:n], X[i])
    for s in range(m + n - 1):
        cells = [(i, s - i) for i in range(m) if 0 <= s - i < n]
        assert sorted(S[s][S[s] != 0]) == sorted(X[i, j] for i, j in cells)
    assert np.array_equal(D.from_skewed(S, m, n), X)


def test_replay_accepts_self_and_catches_a_planted_mistake():
    """The replay follows the given decisions: the recursion's own result is all identical; an
    integer moved by one away from any boundary is a violation; a value exactly on a rounding
    boundary (x = 0.5 in a 1 x 1 problem) accepts both neighbours."""
    X, GA, GB = _problem(5, 4, 16)
    Z, eta, _ = D.gptq2d_buffered(X, GA, GB)
    rep = D.gptq2d_replay(X, GA, GB, Z)
    assert rep["identical"] == 20 and rep["violations"] == 0
    assert np.allclose(rep["eta"], eta, atol=1e-12)
    Y0 = X[0, 0]  # the first cell's pre-round value is X itself
    bad = Z.copy()
    bad[0, 0] += 1 if Y0 - np.rint(Y0) < 0.4 else -1
    assert abs(abs(Y0 - np.rint(Y0)) - 0.5) > 0.05  # the planted move is far from a tie
    assert D.gptq2d_replay(X, GA, GB, bad)["violations"] >= 1
    one = D.gptq2d_replay(np.array([[0.5]]), np.eye(1), np.eye(1), np.array([[1.0]]))
    assert one["in_band"] == 1 and one["violations"] == 0
