"""Parity at full size, in the launch configuration the benchmark times.

H and R are compared in full with the fp64 oracle (computed on the host from the same bf16
bytes); the quantization is checked on sampled rows, which the oracle recomputes one by one
with its own R (rows are independent given R, [T] eq.(7)), by decision replay.
"""
import numpy as np
import pytest
import torch

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

import post_weight_quantization_17_b200 as G  # noqa: E402
from oracle import gptq_oracle as O  # noqa: E402
from tests import _parity as P  # noqa: E402
from workloads.synth import CONFIGS, XSource, make_weight  # noqa: E402


def _oracle_hessian(chunks, d):
    S = np.zeros((d, d))
    n = 0
    for c in chunks:
        for a in range(0, c.shape[0], 16384):
            xc = c[a:a + 16384].float().cpu().double().numpy()
            S += xc.T @ xc
            n += xc.shape[0]
    return (2.0 / n) * S


def _run_full(spec, seed, n_rows=48):
    dev = torch.device("cuda")
    W = make_weight(spec, seed, dev)
    chunks = list(XSource(spec, seed, dev).chunks())
    X = torch.cat(chunks) if len(chunks) > 1 else chunks[0]
    del chunks
    ctx = G.Context(m_max=spec.m, d_max=spec.d, act_order=spec.act_order)
    b = G.LayerBuffers(spec.m, spec.d, spec.bits, spec.group, dev)
    n = G.gptq_hessian_accumulate(ctx, X, b.S, 0)          # one call over every token
    S_gpu = torch.tril(b.S).cpu().double().numpy() * (2.0 / n)
    G.gptq_prepare_hinv(ctx, b.S, n, spec.percdamp, spec.act_order, b.R, b.perm, b.dead)
    G.gptq_quantize_layer(ctx, W, b.R, b.perm if spec.act_order else None, b.dead, spec.bits,
                          spec.group, spec.block, False, b.scales, b.zeros, b.codes, b.W_hat,
                          b.col_loss)
    G.gptq_pack(ctx, b.codes, spec.bits, b.packed)
    G.gptq_sync_status(ctx)
    H = _oracle_hessian([X], spec.d)
    del X
    torch.cuda.empty_cache()
    res = {"H": P.rel_fro(S_gpu, np.tril(H))}
    assert res["H"] <= P.TOL_H, res
    perm_g = b.perm.cpu().numpy().astype(np.int64)
    if spec.act_order:
        assert O.is_valid_act_order(perm_g, H)
    else:
        assert np.array_equal(perm_g, np.arange(spec.d))
    prep = O.prepare_with_retry(H, spec.percdamp, spec.act_order, perm=perm_g)
    Rg = b.R.cpu().double().numpy()
    res["R"] = P.rel_fro(Rg, prep["R"])
    res["Hinv"] = P.rel_fro(Rg.T @ Rg, prep["G"])
    assert res["R"] <= P.TOL_HINV and res["Hinv"] <= P.TOL_HINV, res
    # sampled rows
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(spec.m, size=n_rows, replace=False))
    Wn = W.float().cpu().double().numpy()[rows]
    sc, ze = O.fit_grid(Wn, spec.bits, spec.group)
    assert np.array_equal(b.scales.cpu().numpy()[rows], sc)
    assert np.array_equal(b.zeros.cpu().numpy()[rows], ze)
    Wp = Wn.copy()
    Wp[:, prep["dead"]] = 0.0
    Wp = Wp[:, prep["perm"]]
    gcol = (prep["perm"] // spec.group) if spec.group != -1 else np.zeros(spec.d, np.int64)
    codes = b.codes.cpu().numpy().astype(np.int64)[rows]
    rep = O.decision_replay(Wp, prep["R"], sc, ze, gcol, spec.bits, codes[:, prep["perm"]],
                            band=P.BAND)
    res["identical"] = rep["identical"] / rep["n"]
    res["violations"] = rep["violations"]
    assert rep["violations"] == 0, res
    assert res["identical"] >= P.TOL_CODES_IDENTICAL, res
    inv = np.argsort(prep["perm"])
    res["W_hat"] = P.rel_fro(b.W_hat.cpu().numpy()[rows], rep["replay_Q"][:, inv])
    assert res["W_hat"] <= P.TOL_WHAT, res
    packed = b.packed.cpu().numpy().view(np.uint32)[rows]
    assert np.array_equal(packed, O.pack(codes, spec.bits))
    ctx.close()
    return res


def test_q_proj_4096_full_size():
    res = _run_full(CONFIGS[2][0], seed=1)
    print("q_proj full size:", {k: f"{v:.3e}" if isinstance(v, float) else v for k, v in res.items()})


def test_down_proj_11008_actorder_3bit_full_size():
    res = _run_full(CONFIGS[3][0], seed=2, n_rows=24)
    print("down_proj full size:", {k: f"{v:.3e}" if isinstance(v, float) else v for k, v in res.items()})
