"""Failure detection on the GPU, made on the host: non-finite inputs, an indefinite H, bad
arguments, a too-small workspace.  Nothing here faults, traps or hangs a GPU; each failure is
a status the host reads, and the context stays usable afterwards."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import post_weight_quantization_17_b200 as G  # noqa: E402


@pytest.fixture(scope="module")
def ctx():
    c = G.Context(m_max=64, d_max=128, act_order=True)
    yield c
    c.close()


def _bufs(m, d, bits=4, group=-1):
    return G.LayerBuffers(m, d, bits, group, torch.device("cuda"))


def test_nan_in_X_is_reported(ctx):
    X = torch.randn(50, 16, device="cuda", dtype=torch.bfloat16)
    X[7, 3] = float("nan")
    b = _bufs(8, 16)
    n = G.gptq_hessian_accumulate(ctx, X, b.S, 0)
    with pytest.raises(G.GPTQError) as e:
        G.gptq_prepare_hinv(ctx, b.S, n, 0.01, False, b.R, b.perm, b.dead)
    assert e.value.code == G.GPTQ_ERR_NONFINITE
    _context_still_works(ctx)


def test_inf_in_W_is_reported(ctx):
    b = _bufs(8, 16)
    b.S.copy_(torch.eye(16, device="cuda"))
    G.gptq_prepare_hinv(ctx, b.S, 0, 0.01, False, b.R, b.perm, b.dead)
    W = torch.randn(8, 16, device="cuda", dtype=torch.float16)
    W[2, 5] = float("inf")
    G.gptq_quantize_layer(ctx, W, b.R, None, b.dead, 4, -1, 128, False, b.scales, b.zeros,
                          b.codes, b.W_hat, b.col_loss)
    with pytest.raises(G.GPTQError) as e:
        G.gptq_sync_status(ctx)
    assert e.value.code == G.GPTQ_ERR_NONFINITE
    _context_still_works(ctx)


def test_indefinite_H_retries_then_fails(ctx):
    d = 8
    b = _bufs(4, d)
    # strongly indefinite: damping of 1%..1000% of the mean diagonal cannot fix it
    H = torch.eye(d, device="cuda")
    H[0, 0] = -1000.0
    b.S.copy_(H)
    with pytest.raises(G.GPTQError) as e:
        G.gptq_prepare_hinv(ctx, b.S, 0, 0.01, False, b.R, b.perm, b.dead)
    assert e.value.code == G.GPTQ_ERR_NOT_PD
    # mildly indefinite: fixed after retries with more damping
    H = torch.eye(d, device="cuda") * 2.0
    H[0, 1] = H[1, 0] = 2.05   # eigenvalue -0.05; mean diag 2: λ = 0.002, 0.02 fail, 0.2 works
    b.S.copy_(H)
    lam, retries = G.gptq_prepare_hinv(ctx, b.S, 0, 0.001, False, b.R, b.perm, b.dead)
    assert retries == 2 and abs(lam - 0.2) < 1e-6
    _context_still_works(ctx)


def test_argument_errors(ctx):
    b = _bufs(4, 8)
    W = torch.randn(4, 8, device="cuda", dtype=torch.float16)
    for kw in ({"bits": 0}, {"bits": 9}, {"group": 0}, {"group": -2}, {"block": 0}):
        args = dict(bits=4, group=-1, block=128)
        args.update(kw)
        with pytest.raises(G.GPTQError) as e:
            G.gptq_quantize_layer(ctx, W, b.R, None, b.dead, args["bits"], args["group"],
                                  args["block"], False, b.scales, b.zeros, b.codes, b.W_hat,
                                  b.col_loss)
        assert e.value.code == G.GPTQ_ERR_ARG


def test_workspace_too_small():
    c = G.Context(m_max=4, d_max=8, act_order=False)
    try:
        b = _bufs(256, 512)
        W = torch.randn(256, 512, device="cuda", dtype=torch.float16)
        with pytest.raises(G.GPTQError) as e:
            G.gptq_quantize_layer(c, W, b.R, None, b.dead, 4, -1, 128, False, b.scales,
                                  b.zeros, b.codes, b.W_hat, b.col_loss)
        assert e.value.code == G.GPTQ_ERR_NOMEM
    finally:
        c.close()


def test_wait_budget_runs_out_then_context_recovers():
    """A pipeline wait that runs out: with a one-cycle wait budget the single-SM tensor path of
    the Hessian (128 <= d < 256) gives up at its first wait that is not already satisfied, records
    GPTQ_ERR_TIMEOUT, drains its own copies and tensor-core work, and frees its tensor memory.
    With the default budget restored the same context computes the statistic correctly."""
    c = G.Context(m_max=8, d_max=192, act_order=False)
    try:
        g = torch.Generator(device="cuda").manual_seed(7)
        X = torch.randn(8192, 192, device="cuda", generator=g).to(torch.bfloat16)
        S = torch.zeros(192, 192, device="cuda")
        G.gptq_set_wait_budget(c, 1)
        G.gptq_hessian_accumulate(c, X, S, 0)
        with pytest.raises(G.GPTQError) as e:
            G.gptq_sync_status(c)
        assert e.value.code == G.GPTQ_ERR_TIMEOUT
        G.gptq_set_wait_budget(c, 0)             # back to the default
        n = G.gptq_hessian_accumulate(c, X, S, 0)
        assert G.gptq_sync_status(c) == G.GPTQ_OK and n == 8192
        Xd = X.double()
        ref = torch.tril(Xd.T @ Xd)
        err = (torch.tril(S).double() - ref).norm() / ref.norm()
        assert err <= 1e-4, err
        with pytest.raises(G.GPTQError) as e:
            G.gptq_set_wait_budget(c, -1)
        assert e.value.code == G.GPTQ_ERR_ARG
        _context_still_works(c)
    finally:
        c.close()


def _context_still_works(ctx):
    d = 16
    b = _bufs(8, d)
    b.S.copy_(torch.eye(d, device="cuda") * 3.0)
    G.gptq_prepare_hinv(ctx, b.S, 0, 0.01, False, b.R, b.perm, b.dead)
    W = torch.randn(8, d, device="cuda", dtype=torch.float16) * 0.02
    G.gptq_quantize_layer(ctx, W, b.R, None, b.dead, 4, -1, 128, False, b.scales, b.zeros,
                          b.codes, b.W_hat, b.col_loss)
    assert G.gptq_sync_status(ctx) == G.GPTQ_OK
    assert torch.isfinite(b.W_hat).all()
