"""GPU parity of two-sided rounding (GPTQ-2D) against the oracle's buffered recursion, by decision
replay (the integers are decisions taken in fp32 on the GPU, fp64 in the oracle)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import gptq2d as D  # noqa: E402


@pytest.fixture(scope="module")
def ctx():
    import post_weight_quantization_17_b200 as G
    c = G.Context(m_max=512, d_max=1024, act_order=True)
    yield c
    c.close()


def _pd(k, seed, cond):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.normal(size=(k, k)))
    return (Q * np.geomspace(1.0, 1.0 / cond, k)) @ Q.T


@pytest.mark.parametrize("m,n,cond,seed", [(7, 5, 30, 1), (33, 20, 100, 2), (64, 64, 300, 3),
                                           (130, 70, 1000, 4), (1, 9, 10, 5), (9, 1, 10, 6),
                                           (200, 150, 300, 7), (400, 300, 300, 8)])
def test_twosided_parity(ctx, m, n, cond, seed):
    import post_weight_quantization_17_b200 as G
    rng = np.random.default_rng(seed)
    X = rng.normal(0, 3, (m, n)).astype(np.float32)
    GA = _pd(m, seed + 10, cond).astype(np.float32).astype(np.float64)
    GB = _pd(n, seed + 20, cond).astype(np.float32).astype(np.float64)
    ra = torch.from_numpy(GA.astype(np.float32)).cuda()
    rb = torch.from_numpy(GB.astype(np.float32)).cuda()
    G.gptq_twosided_factor(ctx, ra)
    G.gptq_twosided_factor(ctx, rb)
    RA_o, RB_o = D.factor_upper_inverse(GA), D.factor_upper_inverse(GB)
    for Rg, Ro in ((ra, RA_o), (rb, RB_o)):
        Rg = Rg.cpu().numpy().astype(np.float64)
        assert np.all(np.tril(Rg, -1) == 0)
        assert np.linalg.norm(Rg - Ro) / np.linalg.norm(Ro) <= 1e-4
    Xd = torch.from_numpy(X).cuda()
    Z = torch.full((m, n), float("nan"), device="cuda")
    eta = torch.full((m, n), float("nan"), device="cuda")
    G.gptq_twosided_round(ctx, Xd, ra, rb, Z, eta)
    G.gptq_sync_status(ctx)
    Zg = Z.cpu().numpy().astype(np.float64)
    Eg = eta.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(Zg)) and np.all(Zg == np.rint(Zg))
    rep = D.gptq2d_replay(X.astype(np.float64), GA, GB, Zg, band=1e-3)
    assert rep["violations"] == 0
    assert rep["identical"] / rep["n"] >= 0.999
    assert np.linalg.norm(Eg - rep["eta"]) / max(np.linalg.norm(rep["eta"]), 1e-30) <= 1e-3
    # loss identity on the GPU's own outputs
    loss = D.loss2d(X.astype(np.float64), Zg, GA, GB)
    assert abs(float(np.sum(Eg ** 2)) - loss) <= 1e-3 * loss
