"""gptq_quantize_layer_noalloc — the quantize entry point for callers that cannot allocate device
memory (no context, no workspace; its scratch is a fixed array inside the library) — against
gptq_quantize_layer on the same inputs, on two calls in a row with different layers.

This file is collected last so that a run stopping at the first failure has run every other
test first.  It passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import post_weight_quantization_17_b200 as G  # noqa: E402
from tests import _parity as P  # noqa: E402
from workloads.synth import CONFIGS, LayerSpec  # noqa: E402

LAYERS = [
    CONFIGS[2][0].scaled(200, 640, 3000, chunk=1000),          # 4-bit g128, ragged rows
    LayerSpec("second", 77, 333, 1001, bits=3, group=-1, block=64, act_order=True,
              x_kind="swiglu", x_rank=40, chunk=333),           # act-order, ragged everything
]


def _prepare(ctx, spec, seed):
    W, chunks = P.make_inputs(spec, seed)
    bufs = G.LayerBuffers(spec.m, spec.d, spec.bits, spec.group, W.device)
    n = 0
    for xc in chunks:
        n = G.gptq_hessian_accumulate(ctx, xc, bufs.S, n)
    G.gptq_prepare_hinv(ctx, bufs.S, n, spec.percdamp, spec.act_order, bufs.R, bufs.perm,
                        bufs.dead)
    return W, bufs


def _outputs(spec, device):
    ng = 1 if spec.group == -1 else -(-spec.d // spec.group)
    return dict(scales=torch.full((spec.m, ng), float("nan"), device=device),
                zeros=torch.full((spec.m, ng), -7, dtype=torch.int32, device=device),
                codes=torch.full((spec.m, spec.d), 255, dtype=torch.uint8, device=device),
                W_hat=torch.full((spec.m, spec.d), float("nan"), device=device),
                col_loss=torch.full((spec.d,), float("nan"), device=device))


def test_noalloc_matches_gptq_quantize_layer_on_two_calls():
    ctx = G.Context(m_max=256, d_max=640, act_order=True)
    try:
        for call, (spec, seed) in enumerate(zip(LAYERS, (3, 4))):
            W, bufs = _prepare(ctx, spec, seed)
            perm = bufs.perm if spec.act_order else None
            ref = _outputs(spec, W.device)
            G.gptq_quantize_layer(ctx, W, bufs.R, perm, bufs.dead, spec.bits, spec.group,
                                  spec.block, False, ref["scales"], ref["zeros"], ref["codes"],
                                  ref["W_hat"], ref["col_loss"])
            G.gptq_sync_status(ctx)
            out = _outputs(spec, W.device)
            rc = G.gptq_quantize_layer_noalloc(W, bufs.R, perm, bufs.dead, spec.bits, spec.group,
                                               spec.block, False, out["scales"], out["zeros"],
                                               out["codes"], out["W_hat"], out["col_loss"],
                                               stream=ctx.stream)
            assert rc == G.GPTQ_OK, f"call {call}: status {rc}"
            torch.cuda.synchronize()
            assert torch.equal(out["scales"], ref["scales"]), f"call {call}: scales"
            assert torch.equal(out["zeros"], ref["zeros"]), f"call {call}: zeros"
            # both entry points run the same kernels on the same bytes: bit-equal outputs
            assert torch.equal(out["codes"], ref["codes"]), f"call {call}: codes"
            assert torch.equal(out["W_hat"], ref["W_hat"]), f"call {call}: W_hat"
            assert torch.equal(out["col_loss"], ref["col_loss"]), f"call {call}: col_loss"
    finally:
        ctx.close()


def test_noalloc_rejects_a_layer_larger_than_its_scratch():
    # act-order needs 5 m d bytes of scratch: 2048 x 2048 does not fit in 16 MiB
    m = d = 2048
    dev = torch.device("cuda")
    tiny = torch.zeros(4, dtype=torch.float32, device=dev)
    W = torch.zeros(m, d, dtype=torch.float16, device=dev)
    perm = torch.arange(d, dtype=torch.int32, device=dev)
    rc = G.gptq_quantize_layer_noalloc(W, tiny, perm, None, 4, 128, 128, False, tiny, tiny.int(),
                                       tiny.byte(), tiny, tiny)
    assert rc == G.GPTQ_ERR_ARG
