"""Pins of the CPU oracle against what the source pages and the mathematics fix (no GPU).

Each test ties one oracle function to something other than itself: a worked example printed
by the pages (tests/golden/worked_examples.json, cited there), a closed form, an invariant the
pages prove, a library special case, or brute force on a tiny layer.
"""
import itertools

import numpy as np
import pytest

from oracle import gptq_oracle as O


# ---------------------------------------------------------------- P1: the quantizer
def test_p1_quantizer_example(golden):
    g = golden["P1_quantizer"]
    c, q, u = O.quantize(np.array([g["w"]]), np.float32(g["delta"]), np.int64(g["zero"]), g["bits"])
    assert abs(float(u[0]) - g["u"]) < 1e-6
    assert int(c[0]) == g["code"]
    assert abs(float(q[0]) - g["q"]) < 1e-12


def test_quantizer_clip_and_half_even():
    # clip at both ends, and round-half-to-even at exact ties (fp32-representable ties)
    delta, z = np.float32(0.5), np.int64(2)
    w = np.array([100.0, -100.0, 0.25, 0.75, -0.25])  # u = 200, -200, 0.5, 1.5, -0.5
    c, q, _ = O.quantize(w, delta, z, 2)
    assert list(c) == [3, 0, 2, 4 - 1, 2]  # 0.5->0 (+2), 1.5->2 (+2=4 clipped to 3), -0.5->-0 (+2)
    assert list(q) == [0.5, -1.0, 0.0, 0.5, 0.0]


# ---------------------------------------------------------------- P2: page-1 toy
def test_p2_toy_two_weights(golden):
    g = golden["P2_toy_two_weights"]
    X = np.array(g["X"])
    # the toy uses H = 2 X X^T (no 1/N): hessian() divides by N=2, so scale back
    H = O.hessian(X) * X.shape[1]
    assert np.allclose(H, [[2.08, 0.6], [0.6, 2.5]], atol=1e-12)
    G = np.linalg.inv(H)
    tol = 0.5 * 10 ** -g["printed_digits"]
    assert abs(G[0, 0] - g["Hinv_11"]) <= tol and abs(G[1, 1] - g["Hinv_22"]) <= tol
    w = np.array(g["w"])
    grid = np.array(g["grid"])
    q = grid[np.argmin(np.abs(grid[None, :] - w[:, None]), axis=1)]
    crit = O.obs_criterion(w - q, np.diag(G))
    assert abs(crit[0] - g["criterion_w1"]) <= 5e-5 and abs(crit[1] - g["criterion_w2"]) <= 5e-5
    assert crit[0] < crit[1]  # OBS quantizes w1 first
    delta = O.obs_update(G, 0, w[0] - q[0])
    w_new = w + delta
    assert abs(w_new[0] - q[0]) < 1e-12
    assert abs(w_new[1] - g["w2_after_compensation"]) <= 5e-4
    d_before = np.linalg.norm((w - np.array([q[0], w[1]])) @ X)
    d_after = np.linalg.norm((w - w_new) @ X)
    assert abs(d_before - g["output_distance_before"]) <= 5e-4
    assert abs(d_after - g["output_distance_after"]) <= 5e-4


# ---------------------------------------------------------------- P3: 2-D update, R form
def test_p3_two_dim_update(golden):
    g = golden["P3_two_dim_update"]
    G = np.array(g["G"])
    w = np.array(g["w"])
    rho = w[0] - g["q0"]
    assert abs(rho - g["rho0"]) < 1e-12
    w_after = w + O.obs_update(G, 0, rho)
    assert np.allclose(w_after, g["w_after"], atol=1e-12)
    # R form (eq.(41)/(42)): the explicit recursion's recorded R rows
    _, _, _, Rrows = O.gptq_explicit(w[None, :], G, np.array([[0.25]], np.float32),
                                     np.array([[8]], np.int32), np.array([0, 0]), 4)
    assert np.allclose(Rrows, g["R"], atol=1e-12)
    assert np.allclose(Rrows.T @ Rrows, G, atol=1e-12)
    assert abs(O.downdate(G, 0)[1, 1] - g["next_conditional_G"]) < 1e-12


# ---------------------------------------------------------------- P4: downdate counterexample
def test_p4_downdate(golden):
    g = golden["P4_downdate_counterexample"]
    H = np.array(g["H_F"])
    G = np.linalg.inv(H)
    assert np.allclose(G, g["G_F"], atol=1e-12)
    assert abs(G[1, 1] - g["truncation_wrong"]) < 1e-12
    Gd = O.downdate(G, g["p"])
    assert abs(Gd[1, 1] - g["downdate_right"]) < 1e-12
    assert np.allclose(Gd[0, :], 0) and np.allclose(Gd[:, 0], 0)
    assert abs(Gd[1, 1] - 1.0 / H[1, 1]) < 1e-12  # the inverse of the remaining Hessian


def test_downdate_is_inverse_of_submatrix():
    rng = np.random.default_rng(0)
    A = rng.standard_normal((7, 12))
    H = A @ A.T + 0.1 * np.eye(7)
    G = np.linalg.inv(H)
    for p in range(7):
        keep = [i for i in range(7) if i != p]
        Gd = O.downdate(G, p)
        assert np.allclose(Gd[np.ix_(keep, keep)], np.linalg.inv(H[np.ix_(keep, keep)]),
                           rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- P5: 3-D block constraint
def test_p5_three_dim_block(golden):
    g = golden["P5_three_dim_block"]
    H = np.array(g["H_F"])
    delta, dloss, G_T, T = O.block_constraint_solution(np.linalg.inv(H), g["B"], g["a_B"])
    assert np.allclose(delta, g["delta_star"], atol=1e-12)
    assert abs(dloss - g["dloss"]) < 1e-12
    assert abs(G_T[0, 0] - g["G_T"]) < 1e-12
    # the middle coordinate held at 0 costs more
    d0 = np.array([-1.0, 0.0, -1.0])
    assert abs(0.5 * d0 @ H @ d0 - g["cost_if_middle_fixed"]) < 1e-12


# ---------------------------------------------------------------- P6: full 2x2 layer
def test_p6_full_layer(golden):
    g = golden["P6_full_layer_2x2"]
    X = np.array(g["X"])
    W = np.array(g["W"])
    H = O.hessian(X)
    assert np.allclose(H, g["H"], atol=1e-12)
    grid = (np.full((2, 1), g["delta"], np.float32), np.full((2, 1), g["zero"], np.int32))
    for method in ("explicit", "lazy"):
        out = O.gptq_layer(W, H, g["bits"], -1, block=1 if method == "lazy" else 128,
                           percdamp=0.0, eps=0.0, method=method, grid=grid)
        assert np.allclose(out["G"], g["G"], atol=1e-12)
        assert out["codes"].tolist() == g["K"]
        assert np.allclose(out["W_hat"], g["W_hat"], atol=1e-7)
        # col_loss sums the two rows' per-step losses (each row has the same |rho|)
        tol = 0.5 * 10 ** -g["step_loss_printed_digits"]
        assert np.allclose(out["col_loss"] / 2, g["row_step_losses"], atol=tol)
        le = O.layer_error(W, out["W_hat"], H)
        assert abs(le - g["layer_error"]) <= 0.5 * 10 ** -g["layer_error_printed_digits"]
        assert abs(le - O.layer_error_tokens(W, out["W_hat"], X.T)) < 1e-12
        assert abs(out["col_loss"].sum() - le) < 1e-12  # eq.(67)
    # first column's compensation, as printed in eq.(59)
    Wwork = W.copy()
    rho = Wwork[:, 0] - np.array(g["W_hat"])[:, 0]
    Wwork += O.obs_update(np.array(g["G"]), 0, rho)
    assert np.allclose(Wwork, g["W_work_after_col0"], atol=1e-12)
    # RTN baseline eq.(68)
    c, q = O.quantize_rtn(W, grid[0], grid[1], 4, -1)
    assert np.allclose(q, g["rtn_W"], atol=1e-7)
    assert abs(O.layer_error(W, q, H) - g["rtn_layer_error"]) < 1e-9


# ---------------------------------------------------------------- P9: library special cases
def _spd(d, seed, cond_decay=1e-2):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((d, 3 * d)) * np.logspace(0, np.log10(cond_decay), d)[:, None]
    return O.hessian(A)


def test_p9_hessian_and_inverse_library():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((9, 40))
    assert np.allclose(O.hessian(X), 2.0 / 40 * np.einsum("it,jt->ij", X, X), rtol=1e-13)
    assert np.allclose(O.hessian_tokens(X.T), O.hessian(X), rtol=1e-13)
    H = _spd(30, 4)
    Hl, perm, dead, lam, _ = O.prepare(H, 0.01, False)
    G, R = O.inverse_and_factor(Hl)
    assert np.allclose(G, np.linalg.inv(Hl), rtol=1e-9, atol=1e-12)
    assert np.allclose(R, np.triu(R)) and np.all(np.diag(R) > 0)
    assert np.allclose(R.T @ R, G, rtol=1e-10, atol=1e-12)
    assert np.allclose(R, np.linalg.cholesky(np.linalg.inv(Hl)).T, rtol=1e-8, atol=1e-10)


def test_p7iv_tail_property_and_eq41_rows():
    H = _spd(24, 5)
    Hl, *_ = O.prepare(H, 0.01, False)
    G, R = O.inverse_and_factor(Hl)
    for j in [0, 5, 17, 23]:
        tail = np.linalg.cholesky(np.linalg.inv(Hl[j:, j:])).T
        assert np.allclose(R[j:, j:], tail, rtol=1e-9, atol=1e-11)  # eq.(40)
    W = np.random.default_rng(6).standard_normal((3, 24)) * 0.02
    sc, ze = O.fit_grid(W, 4, -1)
    _, _, _, Rrows = O.gptq_explicit(W, G, sc, ze, np.zeros(24, int), 4)
    assert np.allclose(Rrows, R, rtol=1e-9, atol=1e-11)  # eq.(41) rows from explicit downdates


# ---------------------------------------------------------------- grid fit
def test_grid_fit_closed_form():
    W = np.array([[-0.3, 0.0, 0.45, 0.1], [0.2, 0.4, 0.6, 0.8], [0.0, 0.0, 0.0, 0.0],
                  [-1.0, -0.5, -0.25, -0.75]], np.float32)
    sc, ze = O.fit_grid(W, 4, -1)
    f = np.float32
    assert sc[0, 0] == (f(0.45) - f(-0.3)) / f(15) and ze[0, 0] == int(np.rint(f(0.3) / sc[0, 0]))
    assert sc[1, 0] == f(0.8) / f(15) and ze[1, 0] == 0          # range extended down to 0
    assert sc[2, 0] == 1.0 and ze[2, 0] == 0                      # degenerate range
    assert sc[3, 0] == f(1.0) / f(15) and ze[3, 0] == 15          # range extended up to 0
    # every original weight is representable within half a step (no clipping inside the range)
    for r in range(4):
        c, q, _ = O.quantize(W[r], sc[r, 0], ze[r, 0], 4)
        assert np.all(np.abs(q - W[r]) <= sc[r, 0] / 2 + 1e-7)


def test_grid_fit_groups_and_tail():
    rng = np.random.default_rng(7)
    W = rng.standard_normal((5, 300)).astype(np.float32)
    sc, ze = O.fit_grid(W, 3, 128)
    assert sc.shape == (5, 3)
    for k, (a, b) in enumerate([(0, 128), (128, 256), (256, 300)]):
        s2, z2 = O.fit_grid(W[:, a:b], 3, -1)
        assert np.array_equal(sc[:, k], s2[:, 0]) and np.array_equal(ze[:, k], z2[:, 0])


# ---------------------------------------------------------------- P7 invariants
def _layer(m, d, n, seed, bits=4, group=-1, outliers=True):
    rng = np.random.default_rng(seed)
    F = rng.standard_normal((d, max(2, d // 3)))
    X = F @ rng.standard_normal((F.shape[1], n)) + 0.1 * rng.standard_normal((d, n))
    X *= np.abs(rng.standard_t(3, size=d))[:, None]
    W = rng.standard_normal((m, d)) * 0.02
    if outliers:
        W[:, rng.choice(d, max(1, d // 20), replace=False)] *= 10
    W = W.astype(np.float16).astype(np.float64)
    return W, X


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("group", [-1, 16])
def test_p7i_lazy_equals_unblocked(act_order, group):
    W, X = _layer(12, 48, 200, 11)
    H = O.hessian(X)
    ref = O.gptq_layer(W, H, 3, group, method="explicit", act_order=act_order)
    for block in [1, 5, 16, 48, 100]:
        out = O.gptq_layer(W, H, 3, group, block=block, method="lazy", act_order=act_order)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.allclose(out["W_hat"], ref["W_hat"], atol=1e-12)
        assert np.allclose(out["col_loss"], ref["col_loss"], rtol=1e-8, atol=1e-14)


def test_p7ii_diagonal_hessian_is_rtn():
    W, _ = _layer(9, 20, 10, 12)
    H = np.diag(np.random.default_rng(1).uniform(0.5, 2.0, 20))
    sc, ze = O.fit_grid(W, 4, 8)
    out = O.gptq_layer(W, H, 4, 8, method="explicit")
    c, q = O.quantize_rtn(W, sc, ze, 4, 8)
    assert np.array_equal(out["codes"], c) and np.allclose(out["W_hat"], q)


def test_p7iii_loss_identity():
    W, X = _layer(10, 30, 120, 13)
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 3, -1, method="explicit", percdamp=0.02)
    Hl_orig = np.empty_like(H)
    p = out["perm"]
    Hl_orig[np.ix_(p, p)] = out["H_lambda"]
    dW = W.copy()
    dW[:, out["dead"]] = 0
    assert abs(out["col_loss"].sum() - O.layer_error(dW, out["W_hat"], Hl_orig)) < 1e-10
    # undamped: the recorded losses are the exact layer error (1/N)||ΔW X||^2
    out0 = O.gptq_layer(W, H, 3, -1, method="explicit", percdamp=0.0, eps=0.0)
    assert abs(out0["col_loss"].sum() - O.layer_error_tokens(W, out0["W_hat"], X.T)) < 1e-10


def test_p7v_act_order_identity_and_equivalence():
    W, X = _layer(8, 24, 100, 14)
    H = O.hessian(X)
    # a Hessian whose diagonal is already descending gives π = identity: same as no act-order
    order = np.argsort(-np.diag(H), kind="stable")
    Hs, Ws = H[np.ix_(order, order)], W[:, order]
    a = O.gptq_layer(Ws, Hs, 4, -1, act_order=True)
    b = O.gptq_layer(Ws, Hs, 4, -1, act_order=False)
    assert np.array_equal(a["perm"], np.arange(24))
    assert np.array_equal(a["codes"], b["codes"])
    # eq.(35): permuting W's columns and X's rows leaves W X unchanged
    pi = np.random.default_rng(2).permutation(24)
    assert np.allclose(W[:, pi] @ X[pi, :], W @ X)
    # act-order on a permuted problem gives the permuted answer
    c1 = O.gptq_layer(W, H, 4, -1, act_order=True)
    c2 = O.gptq_layer(W[:, pi], H[np.ix_(pi, pi)], 4, -1, act_order=True)
    assert np.array_equal(c1["codes"][:, pi], c2["codes"])


def test_p7vi_rows_independent_and_vii_landing():
    W, X = _layer(12, 20, 80, 15)
    H = O.hessian(X)
    full = O.gptq_layer(W, H, 4, -1)
    rows = [1, 4, 9]
    sub = O.gptq_layer(W[rows], H, 4, -1, grid=(full["scale"][rows], full["zero"][rows]))
    assert np.array_equal(sub["codes"], full["codes"][rows])
    # each column lands exactly on its grid value: Ŵ = Δ (c - z)
    q = full["scale"][:, [0]] * (full["codes"] - full["zero"][:, [0]])
    assert np.allclose(full["W_hat"], q, atol=1e-7)


def test_dead_features():
    W, X = _layer(6, 10, 40, 16)
    X[[2, 7], :] = 0.0
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 4, -1)
    assert out["dead"].tolist() == [j in (2, 7) for j in range(10)]
    sc, ze = O.fit_grid(W, 4, -1)  # grid fit on the original W (before zeroing)
    assert np.array_equal(out["scale"], sc)
    assert np.allclose(out["W_hat"][:, [2, 7]], 0.0) and np.all(out["codes"][:, [2, 7]] == ze)


def test_retry_raises_damping():
    H = np.array([[1.0, 2.0], [2.0, 1.0]])  # indefinite: eigenvalues 3, -1
    out = O.prepare_with_retry(H, percdamp=0.01)
    assert out["retries"] >= 2 and abs(out["percdamp"] - 0.01 * 10 ** out["retries"]) < 1e-12
    with pytest.raises(np.linalg.LinAlgError):
        O.prepare_with_retry(np.array([[1.0, 0.0], [0.0, -100.0]]), percdamp=0.01)


def test_damping_lambda_hand_values():
    """[T] §10 order (dead features, then the permutation, then damping) and eq.(12): λ is
    percdamp times the mean of diag(H') taken AFTER the dead diagonal entries became 1, with the
    fp32 eps as its floor.  Hand values: diag(H) = (4, 2, 0) -> dead fix-up (4, 2, 1), mean 7/3,
    percdamp 0.03 -> λ = 0.07 (a mean taken before the fix-up would give 0.06)."""
    H = np.array([[4.0, 1.0, 0.0], [1.0, 2.0, 0.0], [0.0, 0.0, 0.0]])
    Hl, perm, dead, lam, Hp = O.prepare(H, 0.03, act_order=True)
    assert abs(lam - 0.07) < 1e-15
    assert dead.tolist() == [False, False, True]
    assert perm.tolist() == [0, 1, 2]               # 4 > 2 > 1 (the dead entry counts as 1)
    assert np.allclose(np.diag(Hl), [4.07, 2.07, 1.07], rtol=0, atol=1e-15)
    assert Hl[0, 1] == 1.0 and Hl[1, 0] == 1.0 and np.all(Hl[2, :2] == 0.0)
    assert np.allclose(Hl - Hp, 0.07 * np.eye(3), rtol=0, atol=1e-15)
    # act-order moves the dead column: diag (1, 5, 0) -> (1, 5, 1), order 1, 0, 2 (stable tie)
    H2 = np.diag([1.0, 5.0, 0.0])
    _, perm2, _, lam2, Hp2 = O.prepare(H2, 0.3, act_order=True)
    assert perm2.tolist() == [1, 0, 2] and np.array_equal(np.diag(Hp2), [5.0, 1.0, 1.0])
    assert abs(lam2 - 0.3 * 7.0 / 3.0) < 1e-15
    # the floor: percdamp 0 (and a percdamp whose λ falls below it) gives exactly 2^-23
    for pd in (0.0, 1e-12):
        assert O.prepare(np.diag([1.0, 1.0]), pd)[3] == 2.0 ** -23
    assert O.FP32_EPS == float(np.finfo(np.float32).eps)


def test_damping_retry_hand_values():
    """The retry reading of [T] §10's remark: percdamp x10 per failed factorization, at most 3
    times.  H = [[1, 1.5], [1.5, 1]] has eigenvalues 2.5 and -0.5 and mean diagonal 1, so
    λ = 0.01 and 0.1 fail and λ = 1 succeeds: two retries, λ = 1.  [[1, 3], [3, 1]] (eigenvalue
    -2) needs λ = 10: three retries.  [[1, 30], [30, 1]] still fails at λ = 10 and raises."""
    out = O.prepare_with_retry(np.array([[1.0, 1.5], [1.5, 1.0]]), percdamp=0.01)
    assert out["retries"] == 2 and abs(out["lam"] - 1.0) < 1e-12
    assert np.allclose(out["H_lambda"], [[2.0, 1.5], [1.5, 2.0]], atol=1e-12)
    out3 = O.prepare_with_retry(np.array([[1.0, 3.0], [3.0, 1.0]]), percdamp=0.01)
    assert out3["retries"] == 3 and abs(out3["lam"] - 10.0) < 1e-9
    with pytest.raises(np.linalg.LinAlgError):
        O.prepare_with_retry(np.array([[1.0, 30.0], [30.0, 1.0]]), percdamp=0.01)


def test_is_valid_act_order_accepts_and_rejects():
    """The parity checker for another implementation's act-order permutation: a descending order
    of diag(H) (dead entries counted as 1), near-ties within rtol in either order, and nothing
    else."""
    H = np.diag([3.0, 0.0, 0.5, 2.0, 2.0 * (1 + 4e-6)])   # dead feature 1 counts as 1
    assert O.is_valid_act_order([0, 4, 3, 1, 2], H)        # exact descending order
    assert O.is_valid_act_order([0, 3, 4, 1, 2], H)        # near-tie (4e-6 < 1e-5) swapped
    assert not O.is_valid_act_order([0, 3, 4, 1, 2], H, rtol=1e-6)  # same swap beyond rtol
    assert not O.is_valid_act_order([0, 4, 3, 2, 1], H)    # 0.5 before the dead entry's 1
    assert not O.is_valid_act_order([4, 0, 3, 1, 2], H)    # 2 before 3: far beyond rtol
    assert not O.is_valid_act_order([0, 4, 4, 1, 2], H)    # repeated index
    assert not O.is_valid_act_order([0, 4, 3, 1], H)       # short list
    assert not O.is_valid_act_order([0, 4, 3, 1, 5], H)    # index out of range
    # it agrees with the oracle's own stable argsort on a random Hessian
    rng = np.random.default_rng(3)
    A = rng.normal(size=(9, 30))
    Hr = A @ A.T
    assert O.is_valid_act_order(O.prepare(Hr, 0.01, True)[1], Hr)
    assert not O.is_valid_act_order(np.arange(9)[::-1].copy(), Hr) or \
        np.all(np.diff(np.diag(Hr)) >= 0)


# ---------------------------------------------------------------- block formula ≡ lazy update
def test_eq32_block_formula_equals_lazy_tail():
    """eq.(32)/(49): D Γ^{-1} G_BT equals E R_BT for a block of already-chosen grid values."""
    H = _spd(14, 17)
    Hl, *_ = O.prepare(H, 0.01, False)
    G, R = O.inverse_and_factor(Hl)
    rng = np.random.default_rng(8)
    Win = rng.standard_normal((4, 14)) * 0.02
    Bn = 5
    Wcur = Win.copy()
    E = np.zeros((4, Bn))
    Q = np.zeros((4, Bn))
    for j in range(Bn):
        Q[:, j] = np.round(Wcur[:, j] / 0.01) * 0.01
        E[:, j] = (Wcur[:, j] - Q[:, j]) / R[j, j]
        Wcur[:, j:Bn] -= np.outer(E[:, j], R[j, j:Bn])
    D = Win[:, :Bn] - Q
    assert np.allclose(D, E @ R[:Bn, :Bn], atol=1e-13)          # eq.(47)
    for r in range(4):
        delta, dloss, _, T = O.block_constraint_solution(G, list(range(Bn)), -D[r])
        assert np.allclose(Win[r] + delta - (Win[r] - E[r] @ R[:Bn, :]), 0, atol=1e-12)


# ---------------------------------------------------------------- P8: brute force
@pytest.mark.parametrize("bits,d,seed", [(2, 1, 0), (2, 4, 1), (3, 4, 2), (2, 6, 3), (3, 5, 4)])
def test_p8_brute_force(bits, d, seed):
    rng = np.random.default_rng(100 + seed)
    n = 3 * d + 2
    X = rng.standard_normal((d, n)) + 0.5 * rng.standard_normal((1, n))
    W = (rng.standard_normal((2, d)) * 0.3).astype(np.float16).astype(np.float64)
    H = O.hessian(X)
    sc, ze = O.fit_grid(W, bits, -1)
    out = O.gptq_layer(W, H, bits, -1, percdamp=0.0, eps=0.0, grid=(sc, ze))
    levels = 2 ** bits
    for r in range(2):
        vals = (sc[r, 0] * (np.arange(levels) - ze[r, 0]).astype(np.float32)).astype(np.float64)
        best = np.inf
        for combo in itertools.product(range(levels), repeat=d):
            dw = W[r] - vals[list(combo)]
            best = min(best, 0.5 * dw @ H @ dw)
        dw = W[r] - out["W_hat"][r]
        gptq_obj = 0.5 * dw @ H @ dw
        assert best <= gptq_obj + 1e-12
        if d == 1:
            assert abs(best - gptq_obj) < 1e-12
        # the last column's choice is the conditional optimum given the earlier codes
        cand = [0.5 * (W[r] - np.r_[out["W_hat"][r, :-1], v]) @ H @ (W[r] - np.r_[out["W_hat"][r, :-1], v])
                for v in vals]
        assert abs(min(cand) - gptq_obj) < 1e-12


# ---------------------------------------------------------------- decision replay
def test_decision_replay_accepts_self_and_flags_planted_mistake():
    W, X = _layer(16, 40, 160, 18)
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 4, 8, method="lazy", block=8)
    codes_p = out["codes"][:, out["perm"]]
    rep = O.decision_replay(out["Wp"], out["R"], out["scale"], out["zero"], out["gcol"], 4, codes_p)
    assert rep["identical"] == rep["n"] and rep["violations"] == 0
    assert np.allclose(rep["replay_loss"][np.argsort(out["perm"])], out["col_loss"], rtol=1e-10)
    assert np.allclose(rep["replay_Q"][:, np.argsort(out["perm"])], out["W_hat"], atol=1e-12)
    assert not rep["rows_with_flips"].any()
    bad = codes_p.copy()
    bad[3, 10] = (bad[3, 10] + 2) % 16
    rep = O.decision_replay(out["Wp"], out["R"], out["scale"], out["zero"], out["gcol"], 4, bad)
    assert rep["violations"] >= 1
    assert rep["rows_with_flips"][3] and rep["rows_with_flips"].sum() == 1


@pytest.mark.parametrize("block,dynamic,act_order", [(8, 0, False), (5, 0, True),
                                                     (16, 8, False), (4, 8, True)])
def test_decision_replay_lazy_blocks_equal_unblocked(block, dynamic, act_order):
    """The lazy-block form of the replay ([T] eq.(46), equal to the unblocked recursion by
    eq.(47)-(49)) takes the same decisions and gives the same Ŵ and loss, also when it follows
    codes with planted mistakes (a flip in band and one far outside) and with R given in fp32."""
    W, X = _layer(12, 40, 200, 21 + block)
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 3, 8, method="lazy", block=8, act_order=act_order,
                       dynamic=bool(dynamic))
    codes_p = out["codes"][:, out["perm"]].copy()
    codes_p[2, 7] = min(codes_p[2, 7] + 1, 7)           # may or may not be in band
    codes_p[5, 21] = (codes_p[5, 21] + 3) % 8            # far outside the band
    for R in (out["R"], out["R"].astype(np.float32)):
        runs = []
        for blk in (0, block):
            if dynamic:
                sc, ze = O.dynamic_grid_arrays(12, 40, dynamic)
            else:
                sc, ze = out["scale"].copy(), out["zero"].copy()
            runs.append(O.decision_replay(out["Wp"], R, sc, ze, out["gcol"], 3, codes_p,
                                          dynamic=dynamic, block=blk,
                                          other_zero=out["zero"] if dynamic else None))
        a, b = runs
        for k in ("n", "identical", "in_band", "violations", "grid_in_band", "grid_violations"):
            assert a[k] == b[k], k
        assert a["violations"] >= 1
        assert np.array_equal(a["rows_with_flips"], b["rows_with_flips"])
        assert np.allclose(a["replay_Q"], b["replay_Q"], rtol=0, atol=1e-12)
        assert np.allclose(a["replay_loss"], b["replay_loss"], rtol=1e-9, atol=0)


# ---------------------------------------------------------------- packing
def test_pack_layout_definition():
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 9]])
    p = O.pack(codes, 4)
    assert p.shape == (1, 2) and p[0, 0] == 0x87654321 and p[0, 1] == 0x9
    codes3 = np.array([[7, 0, 5] + [0] * 7 + [6, 3]])   # 12 codes, 36 bits -> 2 words
    p3 = O.pack(codes3, 3)
    assert p3[0, 0] == (7 | (5 << 6) | (6 << 30)) & 0xFFFFFFFF
    assert p3[0, 1] == ((6 >> 2) | (3 << 1))
    rng = np.random.default_rng(9)
    for bits in (2, 3, 4, 8):
        c = rng.integers(0, 2 ** bits, size=(3, 37))
        assert np.array_equal(O.unpack(O.pack(c, bits), 37, bits), c)
        assert O.pack(c, bits).shape[1] == O.words_per_row(37, bits)


# ---------------------------------------------------------------- dynamic groups ([T] §8.3)
def test_dynamic_one_group_is_the_row_grid():
    """A single dynamic group covering the row is fitted at j = 0 on the untouched working
    weights, i.e. it is the static row grid: identical results."""
    W, X = _layer(8, 24, 100, 21)
    H = O.hessian(X)
    ref = O.gptq_layer(W, H, 4, -1, method="explicit")
    dyn = O.gptq_layer(W, H, 4, 24, method="explicit", dynamic=True)
    assert np.array_equal(dyn["codes"], ref["codes"])
    assert np.array_equal(dyn["W_hat"], ref["W_hat"])
    assert np.array_equal(dyn["scale"], ref["scale"]) and np.array_equal(dyn["zero"], ref["zero"])
    assert np.array_equal(dyn["group_id"], np.zeros(24, np.int64))


@pytest.mark.parametrize("act_order", [False, True])
def test_dynamic_diagonal_hessian_is_rtn_on_processing_groups(act_order):
    """With a diagonal H nothing is compensated, so the working weights never change: each
    dynamic group is the static min-max fit of its processing-order columns and the codes are
    round-to-nearest on that grid.  group_id maps original columns to processing groups."""
    W, _ = _layer(9, 24, 10, 22)
    dg = np.random.default_rng(2).uniform(0.5, 2.0, 24)
    H = np.diag(dg)
    out = O.gptq_layer(W, H, 3, 8, method="explicit", act_order=act_order, dynamic=True)
    perm = out["perm"]
    if act_order:
        assert np.array_equal(perm, np.argsort(-dg, kind="stable"))
    Wp = W[:, perm]
    sc, ze = O.fit_grid(Wp, 3, 8)
    assert np.array_equal(out["scale"], sc) and np.array_equal(out["zero"], ze)
    c, q = O.quantize_rtn(Wp, sc, ze, 3, 8)
    assert np.array_equal(out["codes"][:, perm], c) and np.allclose(out["W_hat"][:, perm], q)
    assert np.array_equal(out["group_id"][perm], np.arange(24) // 8)


@pytest.mark.parametrize("group,blocks", [(4, [1, 2, 4, 8, 12]), (8, [4, 8, 16])])
def test_dynamic_lazy_equals_unblocked(group, blocks):
    """Lazy blocks give the unblocked result when every group starts on a block start or lies
    inside one block ([T] eq.(47)-(49) with the grid refitted from current weights)."""
    W, X = _layer(10, 40, 160, 23)
    H = O.hessian(X)
    ref = O.gptq_layer(W, H, 4, group, method="explicit", act_order=True, dynamic=True)
    for block in blocks:
        out = O.gptq_layer(W, H, 4, group, block=block, method="lazy", act_order=True,
                           dynamic=True)
        assert np.array_equal(out["codes"], ref["codes"]), block
        assert np.array_equal(out["zero"], ref["zero"]), block
        assert np.allclose(out["scale"], ref["scale"], rtol=1e-6), block
        assert np.allclose(out["W_hat"], ref["W_hat"], rtol=1e-6, atol=1e-9), block
    with pytest.raises(ValueError):
        O.gptq_layer(W, H, 4, 8, block=3, method="lazy", dynamic=True)


def test_dynamic_grid_moves_with_compensation():
    """With cross-column compensation the second group's grid is fitted on compensated weights,
    so it differs from the static fit of the original weights (the heuristic the pages warn
    about, [T] §8.4 remark), while the first group's does not."""
    W, X = _layer(6, 16, 80, 24)
    H = O.hessian(X)
    dyn = O.gptq_layer(W, H, 4, 8, method="explicit", dynamic=True)
    sc, ze = O.fit_grid(W, 4, 8)
    assert np.array_equal(dyn["scale"][:, 0], sc[:, 0])
    assert not np.array_equal(dyn["scale"][:, 1], sc[:, 1])


def test_dynamic_replay_accepts_self():
    W, X = _layer(12, 32, 120, 25)
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 4, 8, method="lazy", block=16, act_order=True, dynamic=True)
    codes_p = out["codes"][:, out["perm"]]
    sc, ze = O.dynamic_grid_arrays(12, 32, 8)
    rep = O.decision_replay(out["Wp"], out["R"], sc, ze, out["gcol"], 4, codes_p, dynamic=8)
    assert rep["identical"] == rep["n"] and rep["violations"] == 0
    assert np.array_equal(ze, out["zero"]) and np.allclose(sc, out["scale"], rtol=1e-6)


def test_dynamic_replay_zero_point_decisions():
    """With the other side's zero points given, the replay counts a differing z as in band only
    when it is adjacent and -x_min / Δ sits on the rounding boundary: a row fitted on
    [-1, 5] with 4 bits has Δ = 0.4 and -x_min / Δ = 2.5 exactly, so z = 2 (the oracle's
    ties-to-even) and z = 3 are both correct; a z moved by one anywhere else is a violation."""
    W, _ = _layer(4, 16, 10, 26)
    W[0, :] = np.linspace(-1.0, 5.0, 16)
    H = np.diag(np.linspace(1.0, 2.0, 16))
    out = O.gptq_layer(W, H, 4, 16, method="explicit", dynamic=True)
    assert out["zero"][0, 0] == 2 and out["scale"][0, 0] == np.float32(0.4)
    codes_p = out["codes"][:, out["perm"]]

    def replay(other_zero):
        sc, ze = O.dynamic_grid_arrays(4, 16, 16)
        return O.decision_replay(out["Wp"], out["R"], sc, ze, out["gcol"], 4, codes_p,
                                 dynamic=16, other_zero=other_zero)

    rep = replay(out["zero"])
    assert rep["grid_in_band"] == 0 and rep["grid_violations"] == 0 and rep["violations"] == 0
    tie = out["zero"].copy()
    tie[0, 0] = 3
    rep = replay(tie)
    assert rep["grid_in_band"] == 1 and rep["grid_violations"] == 0
    bad = out["zero"].copy()
    bad[1, 0] += 1 if bad[1, 0] < 15 else -1
    rep = replay(bad)
    assert rep["grid_violations"] == 1


# ------------------------------------------------ grid variants ([T] §1.1, [W] extreme section)
def test_symmetric_grid_worked_values():
    """By hand: a group with max |w| = 0.3 under 4 bits has Δ = 0.6 / 15 = 0.04 and z = 8, so the
    grid is 0.04·{-8..7}; 0.25 / 0.04 = 6.25 rounds to 6 (code 14, value 0.24), and -0.3 / 0.04
    (just below -7.5 in fp32) rounds to -8 (code 0).  An all-zero group gets Δ = 1."""
    W = np.array([[-0.3, 0.1, 0.25, 0.0], [0.0, 0.0, 0.0, 0.0]])
    sc, ze = O.fit_grid_symmetric(W, 15, -1)
    assert sc[0, 0] == np.float32(0.6) / np.float32(15) and ze[0, 0] == 8
    assert sc[1, 0] == 1.0 and ze[1, 0] == 8
    c, q, _ = O.quantize(W[0], sc[0, 0], ze[0, 0], 4)
    assert list(c) == [0, 10, 14, 8]
    assert np.allclose(q, [-0.32, 0.08, 0.24, 0.0], atol=1e-7)


def test_ternary_grid_worked_values():
    """The ternary grid of the extreme-quantization results: Δ = max |w|, z = 1, codes 0..2 in
    2-bit storage, values {-Δ, 0, +Δ}.  w / Δ = 0.52 rounds to 1 (code 2); nothing reaches the
    fourth 2-bit code."""
    w = np.array([[0.5, -0.2, 0.1, -0.05, 0.0, 0.26, -0.5, 0.2]])
    sc, ze = O.fit_grid_symmetric(w, 2, 8)
    assert sc[0, 0] == np.float32(0.5) and ze[0, 0] == 1
    c, q = O.quantize_rtn(w, sc, ze, 2, 8, maxq=2)
    assert list(c[0]) == [2, 1, 1, 1, 1, 2, 0, 1]
    assert set(np.unique(q)) <= {-0.5, 0.0, 0.5}
    # without the level cap a 2-bit code could reach 3 = +2Δ
    c3, _, _ = O.quantize(np.array([1.2]), np.float32(0.5), 1, 2)
    c2, _, _ = O.quantize(np.array([1.2]), np.float32(0.5), 1, 2, maxq=2)
    assert c3[0] == 3 and c2[0] == 2


@pytest.mark.parametrize("kind,bits", [("symmetric", 4), ("symmetric", 3), ("ternary", 2)])
def test_grid_variants_gptq_identities(kind, bits):
    """The recursion's identities hold for the other grids: a diagonal H gives round-to-nearest
    on the grid; lazy blocks give the unblocked result; codes stay within 0..maxq; Ŵ lies on
    the grid."""
    W, X = _layer(10, 32, 128, 27)
    H = O.hessian(X)
    g = 8
    ref = O.gptq_layer(W, H, bits, g, method="explicit", act_order=True, grid_kind=kind)
    maxq = ref["maxq"]
    assert maxq == (2 if kind == "ternary" else 2 ** bits - 1)
    sc, ze = O.fit_grid_symmetric(W, maxq, g)
    assert np.array_equal(ref["scale"], sc) and np.array_equal(ref["zero"], ze)
    assert ref["codes"].min() >= 0 and ref["codes"].max() <= maxq
    gid = np.arange(32) // g
    assert np.allclose(ref["W_hat"], sc[:, gid] * (ref["codes"] - ze[:, gid]), rtol=1e-6)
    for block in (1, 5, 8, 32):
        out = O.gptq_layer(W, H, bits, g, block=block, method="lazy", act_order=True,
                           grid_kind=kind)
        assert np.array_equal(out["codes"], ref["codes"]), block
    dg = np.diag(np.linspace(2.0, 1.0, 32))
    diag = O.gptq_layer(W, dg, bits, g, method="explicit", grid_kind=kind)
    c, _ = O.quantize_rtn(W, sc, ze, bits, g, maxq=maxq)
    assert np.array_equal(diag["codes"], c)
    with pytest.raises(ValueError):
        O.gptq_layer(W, H, 3, g, grid_kind="ternary")


def test_ternary_brute_force_tiny():
    """On a 1 x 4 layer the exhaustive search over the 3^4 ternary code vectors bounds the
    GPTQ layer error from below, and at d = 1 GPTQ attains it (one column is plain rounding,
    which is optimal for a single weight)."""
    rng = np.random.default_rng(28)
    W = rng.normal(0, 0.02, (1, 4))
    X = rng.normal(0, 1, (4, 40))
    H = O.hessian(X)
    out = O.gptq_layer(W, H, 2, -1, method="explicit", grid_kind="ternary")
    sc, ze = out["scale"][0, 0], out["zero"][0, 0]
    best = min(O.layer_error(W, sc * (np.array(cs)[None, :] - ze), H)
               for cs in np.ndindex(3, 3, 3, 3))
    assert O.layer_error(W, out["W_hat"], H) >= best - 1e-15
    W1 = W[:, :1]
    H1 = H[:1, :1]
    one = O.gptq_layer(W1, H1, 2, -1, method="explicit", grid_kind="ternary")
    best1 = min(O.layer_error(W1, one["scale"][0, 0] * (np.array([[c]]) - 1), H1)
                for c in range(3))
    assert np.isclose(O.layer_error(W1, one["W_hat"], H1), best1, rtol=1e-12)


# ------------------------------------------------------------- W4A16 consumer ([T] §1.2, [A])
def test_dequant_matmul_worked_values():
    """By hand: one row of 8 codes 0..7 packed at 4 bits is the word 0x76543210; with Δ = 0.5
    and z = 3 the weights are 0.5·(c - 3) = -1.5, -1, ..., 2; against x = 1..8 the product is
    Σ 0.5 (c - 3)(c + 1) = 0.5 (Σ c² - 2 Σ c - 3·8) = 0.5 (140 - 56 - 24) = 30."""
    packed = np.array([[0x76543210]], np.uint64)
    y = O.dequant_matmul(np.arange(1, 9, dtype=np.float64)[None, :], packed, 8, 4,
                         np.array([[0.5]], np.float32), np.array([[3]]), -1)
    assert y.shape == (1, 1) and y[0, 0] == 30.0


@pytest.mark.parametrize("act_order,dynamic", [(False, False), (True, False), (True, True)])
def test_dequant_matmul_reproduces_layer_output(act_order, dynamic):
    """The packed codes with the layer's grid give back exactly X Ŵᵀ for the Ŵ that the
    quantization returned (static groups indexed by original column; dynamic groups through
    group_id), and at 16 bits of exact weights it is a plain matrix product."""
    W, X = _layer(12, 64, 200, 29)
    H = O.hessian(X)
    g = 16
    out = O.gptq_layer(W, H, 4, g, act_order=act_order, dynamic=dynamic, method="lazy",
                       block=16)
    packed = O.pack(out["codes"], 4)
    Xa = np.random.default_rng(30).normal(size=(5, 64)).astype(np.float32).astype(np.float64)
    y = O.dequant_matmul(Xa, packed, 64, 4, out["scale"], out["zero"], g,
                         group_id=out["group_id"] if dynamic else None)
    assert np.allclose(y, Xa @ out["W_hat"].T, rtol=0, atol=1e-12)
    # an exact identity: Δ = 1, z = 0 and 8-bit codes are the integer matrix itself
    C = np.random.default_rng(31).integers(0, 256, size=(7, 40))
    y8 = O.dequant_matmul(Xa[:, :40], O.pack(C, 8), 40, 8, np.ones((7, 1), np.float32),
                          np.zeros((7, 1), np.int64), -1)
    assert np.array_equal(y8, Xa[:, :40] @ C.T.astype(np.float64))


@pytest.mark.parametrize("bits,group", [(3, 16), (2, 8), (4, -1), (5, 12)])
def test_dequant_matmul_other_widths(bits, group):
    """Codes that straddle 32-bit words (3 and 5 bits) and narrow groups: the product over the
    packed words equals the product over the unpacked code matrix formed directly."""
    rng = np.random.default_rng(32 + bits)
    m, d, T = 9, 70, 4
    codes = rng.integers(0, 2 ** bits, size=(m, d))
    ng = 1 if group == -1 else -(-d // group)
    sc = rng.uniform(0.01, 0.1, (m, ng)).astype(np.float32)
    ze = rng.integers(0, 2 ** bits, (m, ng))
    X = rng.normal(size=(T, d))
    gid = np.zeros(d, np.int64) if group == -1 else np.arange(d) // group
    W_hat = (sc[:, gid] * (codes - ze[:, gid]).astype(np.float32)).astype(np.float32)
    y = O.dequant_matmul(X, O.pack(codes, bits), d, bits, sc, ze, group)
    assert np.allclose(y, X @ W_hat.astype(np.float64).T, rtol=0, atol=1e-12)


def test_tile_codes4_layout():
    """Worked positions of the tile-contiguous layout, its inverse, and its zero padding."""
    rng = np.random.default_rng(40)
    m, d = 130, 288                      # 2 row blocks (the second ragged), 2 column blocks
    packed = rng.integers(1, 2 ** 32, size=(m, d // 8), dtype=np.uint64).astype(np.uint32)
    t = O.tile_codes4(packed, m, d)
    assert t.size == 2 * 2 * 4096
    assert np.array_equal(t[0:32], packed[0, 0:32])            # row 0: no swizzle
    assert np.array_equal(t[32 + 4:32 + 8], packed[1, 0:4])    # row 1, chunk 0 -> position 1
    assert np.array_equal(t[32 * 5 + 4 * 2:32 * 5 + 4 * 3], packed[5, 4 * 7:4 * 8])  # 7 ^ 5 = 2
    assert np.array_equal(t[4096:4096 + 4], packed[0, 32:36])  # column block 1 of row block 0
    # row block 1 holds rows 128, 129 and 126 zero rows; column block 1 holds 4 words per row
    assert np.count_nonzero(t) == np.count_nonzero(packed)
    assert np.array_equal(O.untile_codes4(t, m, d), packed)


def test_gptq_layer_prepare_only_matches_the_full_run():
    W, X = _layer(8, 40, 160, 23)
    H = O.hessian(X)
    full = O.gptq_layer(W, H, 4, 8, method="lazy", block=8, act_order=True)
    prep = O.gptq_layer(W, H, 4, 8, method="prepare", block=8, act_order=True)
    assert prep["codes"] is None and prep["W_hat"] is None and prep["col_loss"] is None
    for k in ("scale", "zero", "perm", "dead", "G", "R", "H_lambda", "Wp", "gcol", "group_id"):
        assert np.array_equal(prep[k], full[k]), k
    assert prep["lam"] == full["lam"] and prep["maxq"] == full["maxq"]
