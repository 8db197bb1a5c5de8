"""GPTQ oracle: a plain, slow, fp64 CPU restatement of GPTQ's layer-wise quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import or call this module.  The product path (the CUDA
library and its Python binding) never touches it, and it shares no code with that path.

Sources, cited by page title and section / equation:

  [T]  "GPTQ 从零推导：4-bit 权重量化为什么能‘量化一列，补偿一列’" (hbblog.cn derivation
       tutorial): §1.1 affine quantizer and min-max fit; eq.(6)-(9) objective and Hessian;
       eq.(12) damping; §4 eq.(22)-(23) single-coordinate update and loss; §6 eq.(26)-(27)
       inverse downdate; §7 eq.(28)-(31) multi-constraint block solution; §8.3 eq.(34)-(35)
       act-order and static groups; eq.(36) quantizer; §9 eq.(37)-(49) Cholesky form and lazy
       blocks; §10 blockwise pseudo-code (order of the preparation steps); §11 worked example.
  [W]  "GPTQ 完全拆解：二阶信息驱动的权重量化，如何把 175B 模型塞进一张 A100"
       (pinghaoyang.com.cn walkthrough): OBS update and greedy criterion, toy example,
       Algorithm 1.
  [A]  "什么是GPTQ（GPTQ）？一种面向生成式预训练 Transformer 的一次性权重量化方法"
       (aiboss88.com wiki), section "工作机制" (how it works): at inference the 4-bit weights
       are dequantized on the fly inside a fused kernel.

Precision: fp64 everywhere, except where floating point decides an integer.  The grid fit
(Δ, z) and each code decision c = clip(rint(w/Δ)+z) are taken in fp32 (IEEE division,
round-half-to-even), which is the precision the CUDA kernels take them in, and Δ is rounded to
fp32 because it is a stored fp32 artifact.

Readings where the pages leave a step open are commented where they show up in the code.  Every function here is pinned by a ``-m "not gpu"``
test (worked examples, closed forms, invariants, library special cases, brute force).
"""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg

FP32_EPS = 2.0 ** -23   # finfo(float32).eps: the damping floor of [T] §10 for an fp32 H


# --------------------------------------------------------------------------------------------
# Hessian
# --------------------------------------------------------------------------------------------
def hessian(X) -> np.ndarray:
    """H = (2/N) X X^T for X [d, N] (feature-major, as [T] §2.1 eq.(5) arranges it).  [T] eq.(9)."""
    X = np.asarray(X, dtype=np.float64)
    n = X.shape[1]
    return (2.0 / n) * (X @ X.T)


def hessian_tokens(Xt) -> np.ndarray:
    """Same H from token-major activations Xt [N, d] (rows are tokens): (2/N) Xt^T Xt."""
    Xt = np.asarray(Xt, dtype=np.float64)
    return (2.0 / Xt.shape[0]) * (Xt.T @ Xt)


# --------------------------------------------------------------------------------------------
# Quantization grid and quantizer
# --------------------------------------------------------------------------------------------
def fit_grid(W, bits: int, group: int):
    """Static min-max affine grid, per row (group == -1) or per (row, group of `group` original
    contiguous columns).  [T] §1.1 (rough min-max fit) and §8.3 (static groups).

    Readings: the fitted range is extended to contain 0, so that the integer zero point z
    represents 0 exactly and lies in [0, 2^b-1]; a degenerate range (all zeros) gets Δ = 1.
    The arithmetic is fp32: Δ = (x_max - x_min) / (2^b - 1), z = clip(rint(-x_min / Δ)).
    Returns scale [m, n_g] float32 and zero [m, n_g] int32.
    """
    W32 = np.asarray(W, dtype=np.float32)
    m, d = W32.shape
    g = d if group == -1 else int(group)
    ng = -(-d // g)
    maxq = np.float32(2 ** bits - 1)
    scale = np.empty((m, ng), np.float32)
    zero = np.empty((m, ng), np.int32)
    for k in range(ng):
        blk = W32[:, k * g:min(d, (k + 1) * g)]
        xmin = np.minimum(blk.min(axis=1), np.float32(0.0))
        xmax = np.maximum(blk.max(axis=1), np.float32(0.0))
        delta = ((xmax - xmin) / maxq).astype(np.float32)
        delta = np.where(xmax == xmin, np.float32(1.0), delta).astype(np.float32)
        z = np.clip(np.rint((-xmin / delta).astype(np.float32)), np.float32(0), maxq)
        scale[:, k] = delta
        zero[:, k] = z.astype(np.int32)
    return scale, zero


def fit_grid_symmetric(W, maxq: int, group: int):
    """Static symmetric grid per row or per (row, group of original columns): the grid is
    centred on 0, which [T] §1.1 mentions beside the min-max fit as a choice real quantizers
    make.  With maxq = 2 it is the ternary grid {-Δ, 0, +Δ} of [W]'s section on extreme
    quantization (2-bit and ternary).

    Readings: M = max |w| over the group; Δ = 2M / maxq (so the codes span [-M, M]); M = 0 gives
    Δ = 1; z = (maxq + 1) // 2 (= 2^(b-1) for maxq = 2^b - 1, 1 for the ternary grid).  fp32
    arithmetic as in `fit_grid`.  Returns scale [m, n_g] float32 and zero [m, n_g] int32.
    """
    W32 = np.asarray(W, dtype=np.float32)
    m, d = W32.shape
    g = d if group == -1 else int(group)
    ng = -(-d // g)
    scale = np.empty((m, ng), np.float32)
    zero = np.full((m, ng), (int(maxq) + 1) // 2, np.int32)
    for k in range(ng):
        M = np.abs(W32[:, k * g:min(d, (k + 1) * g)]).max(axis=1)
        delta = ((np.float32(2.0) * M) / np.float32(maxq)).astype(np.float32)
        scale[:, k] = np.where(M == 0, np.float32(1.0), delta)
    return scale, zero


def _code_max(bits: int, maxq=None) -> int:
    """Largest code: 2^b - 1, unless a grid with fewer levels (the ternary grid: 2) is used."""
    return int(2 ** bits - 1 if maxq is None else maxq)


def quantize(w, delta, zero, bits: int, maxq=None):
    """Affine quantizer of [T] §1.1 / eq.(36): c = clip(round(w/Δ) + z, 0, 2^b - 1),
    q = Δ (c - z).  `maxq` replaces 2^b - 1 for a grid with fewer levels than 2^b.

    The decision is taken in fp32 (w rounded to fp32, IEEE fp32 division, round half to even);
    q is the fp32 product Δ (c - z), returned as fp64.  Returns (c int64, q fp64, u) where
    u = w/Δ (fp32) is the pre-round value.
    """
    w32 = np.asarray(w, dtype=np.float64).astype(np.float32)
    d32 = np.asarray(delta, dtype=np.float32)
    u = (w32 / d32).astype(np.float32)
    c = np.clip(np.rint(u).astype(np.float64) + np.asarray(zero, np.float64), 0,
                _code_max(bits, maxq))
    q = (d32 * (c - zero).astype(np.float32)).astype(np.float32)
    return c.astype(np.int64), q.astype(np.float64), u


def quantize_rtn(W, scale, zero, bits: int, group: int, maxq=None):
    """Round-to-nearest of the original W on the same grid ([T] eq.(68) baseline)."""
    W = np.asarray(W, np.float64)
    m, d = W.shape
    gcol = _group_of_column(np.arange(d), d, group)
    c, q, _ = quantize(W, scale[:, gcol], zero[:, gcol], bits, maxq)
    return c, q


# --------------------------------------------------------------------------------------------
# Preconditioning: dead features, act-order, damping, inverse and its Cholesky factor
# --------------------------------------------------------------------------------------------
def prepare(H, percdamp: float = 0.01, act_order: bool = False, eps: float = FP32_EPS,
            perm=None):
    """The preparation steps of [T] §10 in its order: dead features, then the processing
    permutation, then damping.

    * dead: features with H_jj == 0 get H_jj = 1 (their W columns are zeroed by the caller);
    * act-order: π = stable argsort of diag(H) descending (ties: lower original index first),
      H' = Π H Π^T  ([T] §8.3 eq.(34));
    * damping: λ = max(percdamp * mean(diag H'), eps), H_λ = H' + λ I  ([T] eq.(12), §10).

    `perm` (optional) imposes a processing order instead of computing it; callers use it to
    replay another implementation's act-order permutation after checking that it is a valid
    descending order of diag(H) (near-ties may be ordered either way).

    Returns (H_lambda, perm, dead, lam, H_perm_undamped).
    """
    H = np.array(H, dtype=np.float64, copy=True)
    d = H.shape[0]
    dead = np.diag(H) == 0.0
    idx = np.nonzero(dead)[0]
    H[idx, idx] = 1.0
    if perm is not None:
        perm = np.asarray(perm, dtype=np.int64)
    elif act_order:
        perm = np.argsort(-np.diag(H), kind="stable")
    else:
        perm = np.arange(d)
    Hp = H[np.ix_(perm, perm)]
    lam = max(percdamp * float(np.mean(np.diag(Hp))), eps)
    return Hp + lam * np.eye(d), perm, dead, lam, Hp


def inverse_and_factor(H_lambda):
    """G = H_λ^{-1} and its upper Cholesky factor R (G = R^T R), by the route of [T] §10:
    lower Cholesky L of H_λ, G = (L L^T)^{-1} from L, symmetrise, R = upper Cholesky of G
    ([T] eq.(37)).  Raises numpy.linalg.LinAlgError when H_λ is not positive definite."""
    L = np.linalg.cholesky(H_lambda)
    d = L.shape[0]
    Linv = scipy.linalg.solve_triangular(L, np.eye(d), lower=True)
    G = Linv.T @ Linv
    G = 0.5 * (G + G.T)
    R = np.linalg.cholesky(G).T
    return G, R


def prepare_with_retry(H, percdamp: float = 0.01, act_order: bool = False,
                       eps: float = FP32_EPS, max_retries: int = 3, perm=None):
    """[T] §10 remark: on a failed Cholesky raise the damping and retry.  Reading: percdamp is
    multiplied by 10 per retry, at most `max_retries` times."""
    pd = percdamp
    for attempt in range(max_retries + 1):
        Hl, order, dead, lam, Hp = prepare(H, pd, act_order, eps, perm)
        try:
            G, R = inverse_and_factor(Hl)
            return dict(H_lambda=Hl, H_perm=Hp, perm=order, dead=dead, lam=lam, G=G, R=R,
                        retries=attempt, percdamp=pd)
        except np.linalg.LinAlgError:
            pd *= 10.0
    raise np.linalg.LinAlgError("H_lambda not positive definite after retries")


# --------------------------------------------------------------------------------------------
# Single-coordinate OBS / GPTQ update and the explicit inverse downdate
# --------------------------------------------------------------------------------------------
def obs_update(G_F, p: int, rho):
    """[T] eq.(22): the optimal full update when free coordinate p must move by -rho:
    delta = -(rho / [G_F]_pp) (G_F)_{:,p}.  `rho` may be a vector over rows (then the result is
    [rows, k]).  Returns delta."""
    G_F = np.asarray(G_F, np.float64)
    rho = np.asarray(rho, np.float64)
    return -np.multiply.outer(rho / G_F[p, p], G_F[:, p])


def step_loss(G_F, p: int, rho):
    """[T] eq.(23): minimal added (damped) loss rho^2 / (2 [G_F]_pp)."""
    return np.asarray(rho, np.float64) ** 2 / (2.0 * G_F[p, p])


def obs_criterion(w_err, G_diag):
    """[W] OBS greedy criterion (error^2 / [H^-1]_qq), used only by the toy example."""
    return np.asarray(w_err, np.float64) ** 2 / np.asarray(G_diag, np.float64)


def downdate(G_F, p: int):
    """[T] eq.(26)/(27): inverse of the Hessian with coordinate p removed,
    G_T = (G_F)_TT - (G_F)_Tp (G_F)_pT / [G_F]_pp, returned as the full-size matrix whose row
    and column p are zero (eq.(27))."""
    G_F = np.asarray(G_F, np.float64)
    return G_F - np.outer(G_F[:, p], G_F[p, :]) / G_F[p, p]


def block_constraint_solution(G_F, B, a_B):
    """[T] §7 eq.(29)-(31): with Γ = (G_F)_BB, δ* = (G_F)_{:,B} Γ^{-1} a_B,
    Δℓ* = ½ a_B^T Γ^{-1} a_B, and the next inverse G_T = (G_F)_TT - (G_F)_TB Γ^{-1} (G_F)_BT.
    Returns (delta, dloss, G_T, T)."""
    G_F = np.asarray(G_F, np.float64)
    B = list(B)
    k = G_F.shape[0]
    T = [i for i in range(k) if i not in B]
    Gam = G_F[np.ix_(B, B)]
    y = np.linalg.solve(Gam, np.asarray(a_B, np.float64))
    delta = G_F[:, B] @ y
    dloss = 0.5 * float(np.asarray(a_B, np.float64) @ y)
    Z = np.linalg.solve(Gam, G_F[np.ix_(B, T)])
    G_T = G_F[np.ix_(T, T)] - G_F[np.ix_(T, B)] @ Z
    return delta, dloss, G_T, T


# --------------------------------------------------------------------------------------------
# The column recursion, two ways
# --------------------------------------------------------------------------------------------
def _group_of_column(orig_cols, d: int, group: int):
    """Static group of an original column: floor(col / g) ([T] §8.3), or 0 for a row grid."""
    if group == -1:
        return np.zeros_like(np.asarray(orig_cols))
    return np.asarray(orig_cols) // int(group)


def _dynamic_refit(W, j: int, dyn: int, bits: int, scale, zero):
    """Dynamic groups ([T] §8.3 and §8.4 remark): at a group start j (j % g == 0) the grid of
    processing group j // g is fitted per row, by the same min-max rule as `fit_grid`, on the
    CURRENT working weights of that group's columns W[:, j : j+g] (every earlier column's
    compensation already applied).  Reading: the pages leave the moment open beyond "at the
    start of each group"; the fit sees the group's columns exactly as column j is about to be
    quantized."""
    if dyn > 0 and j % dyn == 0:
        sc, ze = fit_grid(W[:, j:j + dyn], bits, -1)
        scale[:, j // dyn] = sc[:, 0]
        zero[:, j // dyn] = ze[:, 0]


def dynamic_grid_arrays(m: int, d: int, dyn: int):
    """Empty per-(row, processing group) grid arrays for dynamic groups of size dyn."""
    ng = -(-d // dyn)
    return np.zeros((m, ng), np.float32), np.zeros((m, ng), np.int32)


def gptq_explicit(Wp, G, scale, zero, gcol, bits: int, dynamic: int = 0, maxq=None):
    """Unblocked GPTQ with explicit inverse updates, column by column in processing order.

    For j = 0..d-1 over all rows at once (F = {j..d-1}): quantize column j ([T] eq.(36));
    ρ = w_j - q; record the loss Σ_r ρ_r² / (2 G_jj) ([T] eq.(23)); apply eq.(22) to every
    row over the free columns; record the Cholesky row R_{j,j:} = G_{j,j:} / sqrt(G_jj)
    ([T] eq.(41)); downdate G by eq.(27).

    Wp: working weights [m, d] in processing order (dead columns already zero).
    gcol: grid index used at processing position j.  dynamic = g > 0: the grid is refitted at
    every group start by `_dynamic_refit` and written into scale / zero (gcol must be j // g).
    Returns (codes, Q, col_loss, R_rows).
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    G = np.array(G, dtype=np.float64, copy=True)
    m, d = W.shape
    codes = np.zeros((m, d), np.int64)
    Q = np.zeros((m, d), np.float64)
    loss = np.zeros(d, np.float64)
    Rrows = np.zeros((d, d), np.float64)
    for j in range(d):
        _dynamic_refit(W, j, dynamic, bits, scale, zero)
        c, q, _ = quantize(W[:, j], scale[:, gcol[j]], zero[:, gcol[j]], bits, maxq)
        rho = W[:, j] - q
        gjj = G[j, j]
        loss[j] = float(np.sum(step_loss(G, j, rho)))
        # eq.(22) on the free columns j..d-1 (rows/columns < j of G are zero after downdates)
        W[:, j:] += obs_update(G[j:, j:], 0, rho)
        Rrows[j, j:] = G[j, j:] / math.sqrt(gjj)
        G[j:, j:] = downdate(G[j:, j:], 0)
        codes[:, j] = c
        Q[:, j] = q
    return codes, Q, loss, Rrows


def gptq_lazy(Wp, R, scale, zero, gcol, bits: int, block: int, dynamic: int = 0, maxq=None):
    """GPTQ in Cholesky form with lazy block updates: [W] Algorithm 1 / [T] §10 pseudo-code.

    For each block [i, i2): for j in the block quantize column j, η = ρ / R_jj, record
    ρ² / (2 R_jj²) ([T] eq.(43)), update the block's remaining columns by eq.(42) and keep η
    in E; after the block apply W[:, i2:] -= E R[i:i2, i2:] ([T] eq.(46)).
    dynamic = g > 0 refits at group starts as in `gptq_explicit`; the group's columns are then
    current only if every group starts on a block start or lies inside one block
    (g % block == 0 or block % g == 0), which is required.
    Returns (codes, Q, col_loss)."""
    if dynamic > 0 and dynamic % block != 0 and block % dynamic != 0:
        raise ValueError("dynamic groups must start on block starts or lie inside a block")
    W = np.array(Wp, dtype=np.float64, copy=True)
    R = np.asarray(R, np.float64)
    m, d = W.shape
    codes = np.zeros((m, d), np.int64)
    Q = np.zeros((m, d), np.float64)
    loss = np.zeros(d, np.float64)
    for i in range(0, d, block):
        i2 = min(i + block, d)
        # the block's columns as rows (Wb[t] = W[:, i + t]), so that a column is contiguous;
        # E likewise (Eb[t] = η of column i + t)
        Wb = W[:, i:i2].T.copy()
        Eb = np.zeros((i2 - i, m), np.float64)
        for j in range(i, i2):
            t = j - i
            if dynamic > 0 and j % dynamic == 0:
                W[:, i:i2] = Wb.T                        # the refit reads the current columns
            _dynamic_refit(W, j, dynamic, bits, scale, zero)
            c, q, _ = quantize(Wb[t], scale[:, gcol[j]], zero[:, gcol[j]], bits, maxq)
            rho = Wb[t] - q
            eta = rho / R[j, j]
            loss[j] = float(np.sum(rho ** 2)) / (2.0 * R[j, j] ** 2)
            codes[:, j] = c
            Q[:, j] = q
            Eb[t] = eta
            Wb[t:] -= R[j, j:i2, None] * eta[None, :]   # [T] eq.(42) inside the block
        W[:, i:i2] = Wb.T
        W[:, i2:] -= Eb.T @ R[i:i2, i2:]                 # [T] eq.(46)
    return codes, Q, loss


def decision_replay(Wp, R, scale, zero, gcol, bits: int, other_codes, band: float = 1e-3,
                    dynamic: int = 0, other_zero=None, maxq=None, block: int = 0):
    """Check another implementation's codes against this recursion, decision by decision.

    Runs the Cholesky-form recursion ([T] eq.(42)) in fp64 on the same inputs, but at every
    (row, column) it follows `other_codes`.  A decision that differs from this oracle's
    rounding is accepted iff the two codes are adjacent and the oracle's pre-round value w/Δ
    lies within `band` (in units of Δ) of the rounding boundary between them; otherwise it is
    a violation.  Several outputs are correct near a boundary, so the decisions that are
    unique are compared and the rest are checked for validity.

    Along the replayed decisions it also records Ŵ (replay_Q) and the per-column loss
    Σ_r ρ² / (2 R_jj²) ([T] eq.(43)), which are the oracle's values for those decisions.

    block = 0: unblocked, every column's update applied to all later columns at once.  block = B:
    the lazy-block form of [W] Algorithm 1 / [T] §10: updates inside a block of B columns, then
    W[:, i2:] -= E R[i:i2, i2:] ([T] eq.(46)); equal in exact arithmetic ([T] eq.(47)-(49)).  In
    that form R is read one block of rows at a time, so it may be given in fp32 (each block's rows
    are promoted to fp64 when used).

    dynamic = g > 0: the grid is refitted at group starts from the replay's own working
    weights (scale / zero are overwritten), as in `gptq_explicit`.  With `other_zero` (the other
    implementation's zero points, [m, n_groups]) the integer zero point is a decision too: the
    replay follows the other's z, accepting a difference iff the two are adjacent and the
    replay's pre-round value -x_min / Δ lies within `band` of the boundary between them; Δ
    stays the replay's own.  With block > 0 a group must start on a block start or lie inside
    one block.

    Returns dict(n, identical, in_band, violations, max_excess, replay_Q, replay_loss,
    rows_with_flips, grid_in_band, grid_violations).
    """
    if block and dynamic > 0 and dynamic % block != 0 and block % dynamic != 0:
        raise ValueError("dynamic groups must start on block starts or lie inside a block")
    W = np.array(Wp, dtype=np.float64, copy=True)
    if not block:
        R = np.asarray(R, np.float64)
    other = np.asarray(other_codes, np.int64)
    m, d = W.shape
    maxq = _code_max(bits, maxq)
    st = dict(identical=0, in_band=0, violations=0, max_excess=0.0, grid_in_band=0,
              grid_violations=0)
    Qr = np.zeros((m, d), np.float64)
    loss = np.zeros(d, np.float64)
    flipped = np.zeros(m, bool)

    def decide(j, r_jj, wj):
        """Column j (current values wj): follow the other implementation's decision, record
        it, return η."""
        _dynamic_refit(W, j, dynamic, bits, scale, zero)
        if dynamic > 0 and other_zero is not None and j % dynamic == 0:
            k = j // dynamic
            z_o = np.asarray(zero[:, k], np.int64)
            z_g = np.asarray(other_zero, np.int64)[:, k]
            zdiff = z_o != z_g
            if np.any(zdiff):
                # the pre-round value of z as fit_grid forms it (fp32)
                x_min = np.minimum(W[:, j:j + dynamic].astype(np.float32).min(axis=1),
                                   np.float32(0.0))
                t = (-x_min / np.asarray(scale[:, k], np.float32)).astype(np.float32)
                lo = np.minimum(z_o, z_g)[zdiff]
                dist = np.abs(t[zdiff].astype(np.float64) - (lo + 0.5))
                ok = (np.abs(z_o - z_g)[zdiff] == 1) & (dist <= band)
                st["grid_in_band"] += int(np.sum(ok))
                st["grid_violations"] += int(np.sum(~ok))
            zero[:, k] = z_g
        delta = np.asarray(scale[:, gcol[j]], np.float32)
        z = np.asarray(zero[:, gcol[j]], np.int64)
        c_o, _, u = quantize(wj, delta, z, bits, maxq)
        c_g = other[:, j]
        same = c_o == c_g
        st["identical"] += int(np.sum(same))
        diff = ~same
        flipped[diff] = True
        if np.any(diff):
            lo = np.minimum(c_o[diff], c_g[diff])
            adjacent = np.abs(c_o[diff] - c_g[diff]) == 1
            boundary = (lo - z[diff]).astype(np.float64) + 0.5
            dist = np.abs(u[diff].astype(np.float64) - boundary)
            ok = adjacent & (dist <= band) & (lo >= 0) & (lo + 1 <= maxq)
            st["in_band"] += int(np.sum(ok))
            st["violations"] += int(np.sum(~ok))
            if np.any(~ok):
                st["max_excess"] = max(st["max_excess"], float(np.max(dist[~ok])))
        cg = np.clip(c_g, 0, maxq)
        q = (delta * (cg - z).astype(np.float32)).astype(np.float32).astype(np.float64)
        rho = wj - q
        loss[j] = float(np.sum(rho ** 2)) / (2.0 * r_jj ** 2)
        Qr[:, j] = q
        return rho / r_jj

    if not block:
        for j in range(d):
            eta = decide(j, R[j, j], W[:, j])
            W[:, j:] -= np.outer(eta, R[j, j:])
    else:
        for i in range(0, d, block):
            i2 = min(i + block, d)
            Rb = np.asarray(R[i:i2, i:], np.float64)     # this block's rows, columns i..d-1
            # the block's columns as rows (Wb[t] = W[:, i + t]); η likewise
            Wb = W[:, i:i2].T.copy()
            Eb = np.zeros((i2 - i, m), np.float64)
            for j in range(i, i2):
                t = j - i
                if dynamic > 0 and j % dynamic == 0:
                    W[:, i:i2] = Wb.T                    # the refit reads the current columns
                eta = decide(j, Rb[t, t], Wb[t])
                Eb[t] = eta
                Wb[t:] -= Rb[t, t:i2 - i, None] * eta[None, :]
            W[:, i:i2] = Wb.T
            W[:, i2:] -= Eb.T @ Rb[:, i2 - i:]
    return dict(n=m * d, identical=st["identical"], in_band=st["in_band"],
                violations=st["violations"], max_excess=st["max_excess"], replay_Q=Qr,
                replay_loss=loss, rows_with_flips=flipped, grid_in_band=st["grid_in_band"],
                grid_violations=st["grid_violations"])


# --------------------------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------------------------
def gptq_layer(W, H, bits: int, group: int, block: int = 128, percdamp: float = 0.01,
               act_order: bool = False, method: str = "explicit", grid=None,
               eps: float = FP32_EPS, perm=None, dynamic: bool = False,
               grid_kind: str = "minmax"):
    """The layer-wise hot path of [T] §10, end to end on one layer.

    1. grid: fitted on the original W before anything else (static groups), unless given;
    2. prepare: dead features, act-order permutation, damping, G and R (with retry);
    3. working copy W_work = W with dead columns zeroed, permuted into processing order;
    4. the column recursion: `method` = "explicit" (eq.(22)/(26)) or "lazy" (eq.(42)/(46));
       "prepare" stops before it (codes, W_hat and col_loss are None);
    5. un-permute codes, Ŵ and the per-column loss back to original column order.

    dynamic=True (group > 0): dynamic groups ([T] §8.3): the grid of processing group j // g is
    refitted at its start from the current working weights (step 1 is skipped), and the
    returned scale / zero are indexed by processing group; group_id[π_j] = j // g maps each
    original column to its group ([T] §8.3, §8.4 table).

    grid_kind (static groups): "minmax" (`fit_grid`), "symmetric" (`fit_grid_symmetric` with
    maxq = 2^b - 1) or "ternary" (bits = 2, `fit_grid_symmetric` with maxq = 2, codes 0..2).

    Returns a dict with codes [m,d] int64, W_hat [m,d], scale, zero, col_loss [d], perm, dead,
    lam, G, R, H_lambda, Wp (the permuted working copy fed to the recursion), gcol, group_id,
    maxq.
    """
    W = np.asarray(W, np.float64)
    m, d = W.shape
    if dynamic and group <= 0:
        raise ValueError("dynamic groups need group > 0")
    if grid_kind not in ("minmax", "symmetric", "ternary") or (grid_kind == "ternary" and
                                                                 bits != 2):
        raise ValueError(f"grid_kind {grid_kind!r} with bits={bits}")
    maxq = 2 if grid_kind == "ternary" else 2 ** bits - 1
    prep = prepare_with_retry(H, percdamp, act_order, eps, perm=perm)
    perm, dead = prep["perm"], prep["dead"]
    if dynamic:
        scale, zero = dynamic_grid_arrays(m, d, group)
    elif grid is None and grid_kind != "minmax":
        scale, zero = fit_grid_symmetric(W, maxq, group)
    elif grid is None:
        scale, zero = fit_grid(W, bits, group)
    else:
        scale, zero = (np.asarray(grid[0], np.float32), np.asarray(grid[1], np.int32))
    Wwork = W.copy()
    Wwork[:, dead] = 0.0
    Wp = Wwork[:, perm]
    dyn = int(group) if dynamic else 0
    gcol = np.arange(d) // dyn if dynamic else _group_of_column(perm, d, group)
    group_id = np.empty(d, np.int64)
    group_id[perm] = gcol
    if method == "prepare":
        # steps 1-3 only: the grid, the factor and the working copy, for callers that replay
        # another implementation's decisions instead of running the recursion
        return dict(codes=None, W_hat=None, scale=scale, zero=zero, col_loss=None, perm=perm,
                    dead=dead, lam=prep["lam"], G=prep["G"], R=prep["R"],
                    H_lambda=prep["H_lambda"], retries=prep["retries"], Wp=Wp, gcol=gcol,
                    group_id=group_id, maxq=maxq)
    if method == "explicit":
        codes_p, Q_p, loss_p, _ = gptq_explicit(Wp, prep["G"], scale, zero, gcol, bits, dyn,
                                                maxq)
    elif method == "lazy":
        codes_p, Q_p, loss_p = gptq_lazy(Wp, prep["R"], scale, zero, gcol, bits, block, dyn,
                                         maxq)
    else:
        raise ValueError(method)
    codes = np.empty_like(codes_p)
    W_hat = np.empty_like(Q_p)
    col_loss = np.empty_like(loss_p)
    codes[:, perm] = codes_p
    W_hat[:, perm] = Q_p
    col_loss[perm] = loss_p
    return dict(codes=codes, W_hat=W_hat, scale=scale, zero=zero, col_loss=col_loss,
                perm=perm, dead=dead, lam=prep["lam"], G=prep["G"], R=prep["R"],
                H_lambda=prep["H_lambda"], retries=prep["retries"], Wp=Wp, gcol=gcol,
                group_id=group_id, maxq=maxq)


def is_valid_act_order(perm, H, rtol: float = 1e-5) -> bool:
    """True if `perm` lists the columns by descending diag(H) (dead entries counted as 1), up to
    ties within `rtol` relative: the decision taken in another precision may order near-ties
    differently ([T] §8.3: act-order is a heuristic over diag(H))."""
    diag = np.array(np.diag(np.asarray(H, np.float64)), copy=True)
    diag[diag == 0.0] = 1.0
    perm = np.asarray(perm, np.int64)
    if sorted(perm.tolist()) != list(range(len(diag))):
        return False
    v = diag[perm]
    return bool(np.all(v[1:] <= v[:-1] * (1.0 + rtol) + 1e-30))


def layer_error(W, W_hat, H):
    """½ tr(ΔW H ΔW^T), which equals (1/N) ||(W - Ŵ) X||_F^2 when H = 2 X X^T / N
    ([T] eq.(6)-(7), (10))."""
    dW = np.asarray(W, np.float64) - np.asarray(W_hat, np.float64)
    return 0.5 * float(np.sum((dW @ np.asarray(H, np.float64)) * dW))


def layer_error_tokens(W, W_hat, Xt):
    """(1/N) ||(W - Ŵ) X||_F^2 directly from token-major X [N, d] ([T] eq.(6))."""
    dW = np.asarray(W, np.float64) - np.asarray(W_hat, np.float64)
    Y = np.asarray(Xt, np.float64) @ dW.T
    return float(np.sum(Y * Y)) / Xt.shape[0]


# --------------------------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------------------------
def words_per_row(d: int, bits: int) -> int:
    return -(-(d * bits) // 32)


def pack(codes, bits: int):
    """Dense bit-packing of [T] §3.1 ("about md/2 bytes for 4 bit, stored as int32 words").
    Reading (the pages leave the layout to the kernel): per row a little-endian bitstream in
    which code k occupies bits [b*k, b*k + b); word w of the row holds stream bits
    [32w, 32w + 32).  Written from that definition, bit by bit."""
    codes = np.asarray(codes, np.int64)
    m, d = codes.shape
    nw = words_per_row(d, bits)
    out = np.zeros((m, nw), np.uint64)
    for k in range(d):
        for t in range(bits):
            bit = (codes[:, k] >> t) & 1
            pos = bits * k + t
            out[:, pos // 32] |= (bit.astype(np.uint64) << np.uint64(pos % 32))
    return out.astype(np.uint32)


def unpack(packed, d: int, bits: int):
    """Inverse of `pack`."""
    packed = np.asarray(packed, np.uint64)
    m = packed.shape[0]
    codes = np.zeros((m, d), np.int64)
    for k in range(d):
        for t in range(bits):
            pos = bits * k + t
            bit = (packed[:, pos // 32] >> np.uint64(pos % 32)) & np.uint64(1)
            codes[:, k] |= (bit.astype(np.int64) << t)
    return codes


# --------------------------------------------------------------------------------------------
# Consumer of the packed format: the W4A16 product
# --------------------------------------------------------------------------------------------
def dequant_matmul(X, packed, d: int, bits: int, scale, zero, group: int, group_id=None):
    """Y = X Ŵᵀ for 16-bit activations and the packed codes, the product a W4A16 layer computes
    at inference ([T] §1.2: weights stored as codes, activations kept in FP16/BF16; [A] "how it
    works": the codes are dequantized inside the fused kernel).

    X [T, d] (token-major), packed [m, words] in the layout of `pack`, scale [m, n_g] fp32,
    zero [m, n_g].  The weight is the quantizer's output Ŵ[r, k] = Δ[r, g(k)] (c[r, k] -
    z[r, g(k)]) in fp32 ([T] eq.(36), §8.4), with g(k) = group_id[k] when given (dynamic groups
    under act-order, [T] §8.4 table) else k // group (static groups; 0 for group = -1).
    Returns Y [T, m] in fp64 (X and Ŵ taken exactly, products and sums in fp64).
    """
    codes = unpack(packed, d, bits)
    if group_id is not None:
        gid = np.asarray(group_id, np.int64)
    elif group == -1:
        gid = np.zeros(d, np.int64)
    else:
        gid = np.arange(d) // int(group)
    sc = np.asarray(scale, np.float32)[:, gid]
    ze = np.asarray(zero, np.int64)[:, gid]
    W_hat = (sc * (codes - ze).astype(np.float32)).astype(np.float32)
    return np.asarray(X, np.float64) @ W_hat.astype(np.float64).T


def tile_codes4(packed, m: int, d: int):
    """The tile-contiguous layout of 4-bit packed codes that the library's product can read with
    whole-tile copies (a layout of this library; the pages fix none for deployed codes): 16 KB
    tiles of 128 rows x 256 codes, tiles in row-major order of (row block, column block); inside a
    tile row r takes 128 bytes and its 16-byte chunk c (32 codes, words 4c .. 4c + 3 of the
    block) sits at position c XOR (r mod 8).  Rows and columns past the matrix are zero.
    Returns a flat uint32 array."""
    packed = np.asarray(packed, np.uint32)
    wpr = d // 8
    RT, KT = -(-m // 128), -(-d // 256)
    full = np.zeros((RT * 128, KT * 32), np.uint32)
    full[:m, :wpr] = packed[:, :wpr]
    t = full.reshape(RT, 128, KT, 8, 4).transpose(0, 2, 1, 3, 4)    # [RT, KT, r, c, word]
    r = np.arange(128)[:, None]
    logical = np.arange(8)[None, :] ^ (r & 7)                      # chunk stored at pc
    out = np.take_along_axis(t, logical[None, None, :, :, None], axis=3)
    return out.reshape(-1)


def untile_codes4(tiled, m: int, d: int):
    """Inverse of `tile_codes4` (the [m, d / 8] packed words)."""
    RT, KT = -(-m // 128), -(-d // 256)
    t = np.asarray(tiled, np.uint32).reshape(RT, KT, 128, 8, 4)
    r = np.arange(128)[:, None]
    stored_at = np.arange(8)[None, :] ^ (r & 7)                    # where logical chunk c sits
    logical = np.take_along_axis(t, stored_at[None, None, :, :, None], axis=3)
    full = logical.transpose(0, 2, 1, 3, 4).reshape(RT * 128, KT * 32)
    return full[:m, :d // 8]
