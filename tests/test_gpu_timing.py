"""The per-stage timing facility (gptq_timing_enable / gptq_timing_read) that the bench's stage
rooflines read.  With timing on, every stage of the hot path is counted with the expected number
of launches.  The stage times add up to no more than the elapsed time of the calls, since timed
launches run one after another on the context stream, the factorization included.  The results
are bit-identical to a run without timing."""
import pytest
import torch

pytestmark = pytest.mark.gpu

import post_weight_quantization_17_b200 as G  # noqa: E402

M, D, N = 512, 4096, 8192   # d = 4096: the factorization's top node runs on CTA pairs


def _layer(ctx, X, W, b):
    """The whole hot path once; returns its elapsed time on the context stream (ms)."""
    s = ctx.stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    n = G.gptq_hessian_accumulate(ctx, X, b.S, 0)
    G.gptq_prepare_hinv(ctx, b.S, n, 0.01, False, b.R, b.perm, b.dead)
    G.gptq_quantize_layer(ctx, W, b.R, None, b.dead, 4, 128, 128, 0, b.scales, b.zeros, b.codes,
                          b.W_hat, b.col_loss)
    G.gptq_pack(ctx, b.codes, 4, b.packed)
    e1.record(s)
    G.gptq_sync_status(ctx)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def test_stage_timing_counts_every_stage_and_changes_nothing():
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(3)
    X = torch.randn(N, D, device=dev, generator=g).to(torch.bfloat16)
    W = (torch.randn(M, D, device=dev, generator=g) * 0.02).half()
    stream = torch.cuda.Stream(dev)
    ctx = G.Context(m_max=M, d_max=D, act_order=False, stream=stream)
    try:
        plain = G.LayerBuffers(M, D, 4, 128, dev)
        timed = G.LayerBuffers(M, D, 4, 128, dev)
        _layer(ctx, X, W, plain)                       # warm-up, also the reference results

        G.gptq_timing_enable(ctx, True)
        elapsed = _layer(ctx, X, W, timed)
        stages = G.gptq_timing_read(ctx)
        assert G.gptq_timing_read(ctx) == {}           # the records were dropped
        G.gptq_timing_enable(ctx, False)

        for name in ("hessian", "prepare", "factor_base", "factor_gemm", "factor_copy", "grid",
                     "column", "update", "output", "pack"):
            assert name in stages, name
            ms, launches = stages[name]
            assert ms >= 0.0 and launches > 0, (name, stages[name])
        assert stages["hessian"][1] == 1
        assert stages["factor_base"][1] == D // 128    # one base block per 128 features
        assert stages["column"][1] >= D // 128         # a column kernel per 128-column block
        assert stages["pack"][1] == 1
        total = sum(ms for ms, _ in stages.values())
        assert total <= elapsed * 1.02 + 0.05, (total, elapsed, stages)

        for name in ("S", "R", "perm", "dead", "scales", "zeros", "codes", "W_hat", "col_loss",
                     "packed"):
            assert torch.equal(getattr(plain, name), getattr(timed, name)), name
    finally:
        ctx.close()
