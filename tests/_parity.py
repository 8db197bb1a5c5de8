"""Helpers shared by the GPU parity tests: run one layer through the C ABI step by step, run the
oracle on the same bytes, and compare with the tolerances of the hot-path contract:

  H and H^-1 (and R) within 1e-4 relative Frobenius; codes identical for >= 99.9% of weights with
  every mismatch within 1e-3·Δ of a rounding boundary (decision replay); Ŵ within 1e-3
  relative; layer error within 1% of the oracle's; grid (Δ, z) and packed words bit-exact.

Ŵ and the per-column loss are compared with the oracle's values for the same decisions (the
replay): one legitimate boundary flip moves the rest of its row by whole grid steps, so a
free-running comparison measures how many rows flipped, not the arithmetic.  Rows whose
decisions all agree are also compared with the free-running oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import post_weight_quantization_17_b200 as G
from oracle import gptq_oracle as O
from workloads import synth

TOL_H = 1e-4
TOL_HINV = 1e-4
TOL_CODES_IDENTICAL = 0.999
BAND = 1e-3
TOL_WHAT = 1e-3
TOL_LAYER_ERR = 0.01


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def make_inputs(spec: synth.LayerSpec, seed: int, zero_features=()):
    W = synth.make_weight(spec, seed, "cuda")
    xs = synth.XSource(spec, seed, "cuda")
    chunks = []
    for c in xs.chunks():
        if zero_features:
            c[:, list(zero_features)] = 0
        chunks.append(c)
    return W, chunks


def gpu_run(ctx, spec, W, chunks, block=None, H32=None, grid_given=0, grid=None):
    """Runs the four ABI calls; returns numpy copies of every output plus the raw S.  grid =
    (scales, zeros) hands the library a caller-chosen grid (grid_given = 1)."""
    m, d = W.shape
    bufs = G.LayerBuffers(m, d, spec.bits, spec.group, W.device)
    if grid is not None:
        bufs.scales.copy_(torch.as_tensor(grid[0]))
        bufs.zeros.copy_(torch.as_tensor(grid[1]))
        grid_given = 1
    n = 0
    S_raw = None
    if H32 is None:
        for xc in chunks:
            n = G.gptq_hessian_accumulate(ctx, xc, bufs.S, n)
        S_raw = bufs.S.clone()
    else:
        bufs.S.copy_(torch.as_tensor(H32, device=W.device))
    lam, retries = G.gptq_prepare_hinv(ctx, bufs.S, n, spec.percdamp, spec.act_order, bufs.R,
                                       bufs.perm, bufs.dead)
    G.gptq_quantize_layer(ctx, W, bufs.R, bufs.perm if spec.act_order else None, bufs.dead,
                          spec.bits, spec.group, block or spec.block, grid_given, bufs.scales,
                          bufs.zeros, bufs.codes, bufs.W_hat, bufs.col_loss)
    G.gptq_pack(ctx, bufs.codes, spec.bits, bufs.packed)
    G.gptq_sync_status(ctx)
    torch.cuda.synchronize()
    out = {k: getattr(bufs, k).cpu().numpy() for k in
           ("R", "perm", "dead", "scales", "zeros", "codes", "W_hat", "col_loss", "packed")}
    out["S_raw"] = None if S_raw is None else S_raw.cpu().numpy()
    out["n"] = n
    out["lam"] = lam
    out["retries"] = retries
    return out


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_hessian(gpu, Xt):
    """GPU H (lower triangle of 2 S / N) against the oracle's fp64 H."""
    H = O.hessian_tokens(Xt)
    Hg = np.tril(gpu["S_raw"].astype(np.float64)) * (2.0 / gpu["n"])
    err = rel_fro(Hg, np.tril(H))
    assert err <= TOL_H, f"H rel err {err:.3e}"
    return H, err


TOL_DYN_SCALE = 1e-4


def check_layer(gpu, Wn, H, spec, block=None, method="explicit", dynamic=False, grid=None,
                grid_kind="minmax", replay_block=0, free_running=True):
    """Oracle on the same H and W; returns a dict of the measured discrepancies after
    asserting the contract's tolerances.  replay_block > 0 replays the decisions in the
    lazy-block form (for large layers; same decisions as the unblocked replay).
    free_running=False skips the oracle's own recursion: the decisions, Ŵ and the per-column loss
    are then checked against the replay only (not the free-running Ŵ and layer error).

    dynamic: the GPU ran with dynamic groups (grid_given = 2).  Each group's grid is then fitted
    on weights that already carry fp32 compensation, so Δ is compared with the replay's own fit
    within TOL_DYN_SCALE (relative) and z is a decision the replay follows like the codes."""
    perm_g = gpu["perm"].astype(np.int64)
    perm = None
    if spec.act_order:
        perm_o = np.argsort(-np.where(np.diag(H) == 0, 1.0, np.diag(H)), kind="stable")
        if not np.array_equal(perm_g, perm_o):
            assert O.is_valid_act_order(perm_g, H), "GPU act-order permutation is not a valid order"
        perm = perm_g
    else:
        assert np.array_equal(perm_g, np.arange(H.shape[0]))
    o = O.gptq_layer(Wn, H, spec.bits, spec.group, block or spec.block, spec.percdamp,
                     spec.act_order, method=method if free_running else "prepare", perm=perm,
                     dynamic=dynamic, grid=grid, grid_kind=grid_kind)
    res = {}
    if not dynamic:
        # grid: bit-exact (both sides decide in fp32 on the same fp16 values)
        assert np.array_equal(gpu["scales"], o["scale"]), "scales differ"
        assert np.array_equal(gpu["zeros"], o["zero"]), "zeros differ"
    assert np.array_equal(gpu["dead"].astype(bool), o["dead"])
    # R and H^-1 = R^T R
    Rg = gpu["R"].astype(np.float64)
    assert np.all(np.tril(Rg, -1) == 0)
    res["R"] = rel_fro(Rg, o["R"])
    res["Hinv"] = rel_fro(Rg.T @ Rg, o["G"])
    assert res["R"] <= TOL_HINV and res["Hinv"] <= TOL_HINV, res
    # codes: decision replay in processing order
    codes_p = gpu["codes"].astype(np.int64)[:, o["perm"]]
    if dynamic:
        sc_r, ze_r = O.dynamic_grid_arrays(*o["Wp"].shape, spec.group)
        rep = O.decision_replay(o["Wp"], o["R"], sc_r, ze_r, o["gcol"], spec.bits, codes_p,
                                band=BAND, dynamic=spec.group, other_zero=gpu["zeros"])
        res["grid_scale_rel"] = float(np.max(np.abs(gpu["scales"].astype(np.float64) - sc_r) /
                                             sc_r))
        res["grid_zero_flips"] = rep["grid_in_band"]
        assert rep["grid_violations"] == 0, f"{rep['grid_violations']} zero points outside the band"
        assert res["grid_scale_rel"] <= TOL_DYN_SCALE, res
    else:
        rep = O.decision_replay(o["Wp"], o["R"], o["scale"], o["zero"], o["gcol"], spec.bits,
                                codes_p, band=BAND, maxq=o["maxq"], block=replay_block)
    res["identical"] = rep["identical"] / rep["n"]
    res["in_band"] = rep["in_band"]
    res["violations"] = rep["violations"]
    assert rep["violations"] == 0, f"{rep['violations']} code decisions outside the band"
    assert res["identical"] >= TOL_CODES_IDENTICAL, res
    # Ŵ against the replay (same decisions) and, on rows without flips, the free-running oracle
    inv = np.argsort(o["perm"])
    Q_replay = rep["replay_Q"][:, inv]
    res["W_hat"] = rel_fro(gpu["W_hat"], Q_replay)
    assert res["W_hat"] <= TOL_WHAT, res
    clean = ~rep["rows_with_flips"]
    res["rows_with_flips"] = int(np.sum(~clean))
    if free_running:
        if np.any(clean):
            res["W_hat_clean_rows"] = rel_fro(gpu["W_hat"][clean], o["W_hat"][clean])
            assert res["W_hat_clean_rows"] <= TOL_WHAT, res
        # layer error of the free-running outputs
        e_g = O.layer_error(Wn, gpu["W_hat"], H)
        e_o = O.layer_error(Wn, o["W_hat"], H)
        res["layer_err"] = abs(e_g - e_o) / e_o if e_o > 0 else abs(e_g)
        assert res["layer_err"] <= TOL_LAYER_ERR, res
    # per-column loss ([T] eq.(43)) against the replay's
    res["col_loss"] = rel_fro(gpu["col_loss"], rep["replay_loss"][inv])
    assert res["col_loss"] <= 1e-3, res
    # Ŵ is exactly Δ (c - z) in fp32
    gcol_orig = o["gcol"][np.argsort(o["perm"])]
    sc = gpu["scales"][:, gcol_orig]
    ze = gpu["zeros"][:, gcol_orig]
    q = (sc * (gpu["codes"].astype(np.int64) - ze).astype(np.float32)).astype(np.float32)
    assert np.array_equal(q, gpu["W_hat"]), "W_hat is not Δ (c - z)"
    # packing: bit-exact against the oracle's definition of the layout
    assert np.array_equal(gpu["packed"].view(np.uint32), O.pack(gpu["codes"], spec.bits))
    return res
