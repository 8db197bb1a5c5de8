"""GPU parity: the C-ABI path against the fp64 oracle on the same seeded inputs, at sizes the
oracle finishes in seconds that still span several tiles and ragged tails."""
import dataclasses

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from tests import _parity as P  # noqa: E402
from workloads.synth import CONFIGS, LayerSpec  # noqa: E402


@pytest.fixture(scope="module")
def ctx():
    import post_weight_quantization_17_b200 as G
    c = G.Context(m_max=512, d_max=1024, act_order=True)  # Hessian-only calls need no workspace
    yield c
    c.close()


SMALL = [
    ("config1_tiny", CONFIGS[1][0], 0),
    ("qproj_shape", CONFIGS[2][0].scaled(160, 384, 3000, chunk=1024), 1),
    ("downproj_actorder_3bit", CONFIGS[3][0].scaled(96, 300, 2000, chunk=700), 2),
    ("block7b_down_shape", CONFIGS[4][6].scaled(72, 256, 1500), 3),
    ("fc2_shape_2bit", CONFIGS[5][1].scaled(130, 256, 2048, chunk=512), 4),
    ("fc2_shape_4bit", CONFIGS[5][0].scaled(40, 200, 900, chunk=300), 9),
    # m >= 256 and tails past the first super-block: the split-operand pair GEMM (ragged rows,
    # a 588-column tail) and, for the last 76 columns, the single-CTA GEMM
    ("pair_tail_ragged", CONFIGS[2][0].scaled(300, 1100, 2500, chunk=1000), 10),
    ("ragged_all", LayerSpec("ragged", 77, 333, 1001, bits=4, group=128, block=128,
                             act_order=False, x_kind="lowrank_t3", x_rank=40, chunk=333), 5),
    ("ragged_actorder_rowgrid", LayerSpec("ragged2", 33, 197, 517, bits=3, group=-1, block=64,
                                          act_order=True, x_kind="swiglu", x_rank=30,
                                          chunk=200), 6),
    ("degenerate_1x1", LayerSpec("one", 1, 1, 1, bits=4, group=-1, block=128, act_order=False,
                                 x_kind="lowrank_t3", x_rank=1, chunk=1), 7),
    ("tiny_3x5", LayerSpec("tiny35", 3, 5, 4, bits=2, group=2, block=2, act_order=True,
                           x_kind="relu_lowrank", x_rank=2, chunk=3), 8),
]


@pytest.mark.parametrize("name,spec,seed", SMALL, ids=[c[0] for c in SMALL])
def test_layer_parity(ctx, name, spec, seed):
    W, chunks = P.make_inputs(spec, seed)
    gpu = P.gpu_run(ctx, spec, W, chunks)
    Xt = torch.cat(chunks).cpu().double().numpy()
    Wn = P.to_np64(W)
    H, herr = P.check_hessian(gpu, Xt)
    res = P.check_layer(gpu, Wn, H, spec)
    print(name, f"H={herr:.2e}", {k: (f"{v:.2e}" if isinstance(v, float) else v) for k, v in res.items()})


STATIC_MORE = [
    # 32-column groups with 2 bits: several grids inside one column-kernel block
    ("static_g32_2bit", dataclasses.replace(
        CONFIGS[5][1].scaled(130, 256, 2048, chunk=512), group=32), 12),
    # 8-column groups under act-order: the per-column grid lookup of the general path
    ("static_g8_actorder", dataclasses.replace(
        CONFIGS[3][0].scaled(64, 200, 1500, chunk=500), group=8, bits=4), 13),
]


@pytest.mark.parametrize("name,spec,seed", STATIC_MORE, ids=[c[0] for c in STATIC_MORE])
def test_static_small_groups_parity(ctx, name, spec, seed):
    W, chunks = P.make_inputs(spec, seed)
    gpu = P.gpu_run(ctx, spec, W, chunks)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, herr = P.check_hessian(gpu, Xt)
    res = P.check_layer(gpu, P.to_np64(W), H, spec)
    print(name, f"H={herr:.2e}", {k: (f"{v:.2e}" if isinstance(v, float) else v) for k, v in res.items()})


@pytest.mark.parametrize("act_order", [False, True])
def test_given_symmetric_grid_parity(ctx, act_order):
    """grid_given = 1: a caller-chosen grid (here symmetric, z = 2^(b-1), Δ = 2 max|w| / maxq
    per row and group of 128) is used as is and returned untouched."""
    spec = dataclasses.replace(CONFIGS[2][0].scaled(96, 384, 2000, chunk=1000),
                               act_order=act_order)
    W, chunks = P.make_inputs(spec, 14)
    Wn = P.to_np64(W)
    maxq = 2 ** spec.bits - 1
    amax = np.abs(Wn.astype(np.float32)).reshape(96, -1, 128).max(axis=2)
    scales = np.where(amax > 0, 2 * amax / np.float32(maxq), 1).astype(np.float32)
    zeros = np.full(scales.shape, (maxq + 1) // 2, np.int32)
    gpu = P.gpu_run(ctx, spec, W, chunks, grid=(scales, zeros))
    assert np.array_equal(gpu["scales"], scales) and np.array_equal(gpu["zeros"], zeros)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, _ = P.check_hessian(gpu, Xt)
    res = P.check_layer(gpu, Wn, H, spec, grid=(scales, zeros))
    print("given_grid", act_order, res)


GRID_VARIANTS = [
    # symmetric 4-bit g128 under act-order (grid_given = 3)
    ("symmetric_4bit_g128", dataclasses.replace(
        CONFIGS[2][0].scaled(160, 384, 3000, chunk=1024), act_order=True), 15, 3, "symmetric"),
    # symmetric 3-bit per row, ragged
    ("symmetric_3bit_row_ragged", LayerSpec("sym3", 77, 333, 1001, bits=3, group=-1, block=128,
                                            act_order=False, x_kind="lowrank_t3", x_rank=40,
                                            chunk=333), 16, 3, "symmetric"),
    # the ternary grid at g = 8 (grid_given = 4), the extreme case of the results
    ("ternary_g8", dataclasses.replace(
        CONFIGS[5][1].scaled(130, 256, 2048, chunk=512), group=8), 17, 4, "ternary"),
    ("ternary_g8_actorder_ragged", dataclasses.replace(
        CONFIGS[3][0].scaled(61, 203, 1500, chunk=500), group=8, bits=2), 18, 4, "ternary"),
]


@pytest.mark.parametrize("name,spec,seed,mode,kind", GRID_VARIANTS,
                         ids=[c[0] for c in GRID_VARIANTS])
def test_grid_variants_parity(ctx, name, spec, seed, mode, kind):
    """Symmetric and ternary static grids fitted on the GPU, then the same recursion."""
    W, chunks = P.make_inputs(spec, seed)
    gpu = P.gpu_run(ctx, spec, W, chunks, grid_given=mode)
    if kind == "ternary":
        assert gpu["codes"].max() <= 2 and np.all(gpu["zeros"] == 1)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, herr = P.check_hessian(gpu, Xt)
    res = P.check_layer(gpu, P.to_np64(W), H, spec, grid_kind=kind)
    print(name, f"H={herr:.2e}", {k: (f"{v:.2e}" if isinstance(v, float) else v) for k, v in res.items()})


DYNAMIC = [
    # g = 128: one grid per kernel block, fitted from the staged block; ragged last group
    ("dyn128_qproj_shape", CONFIGS[2][0].scaled(160, 600, 3000, chunk=1024), 1, 128),
    # g = 32: one grid per sub-block, with act-order and 3 bits; ragged rows and last group
    ("dyn32_downproj_actorder", dataclasses.replace(
        CONFIGS[3][0].scaled(77, 300, 2000, chunk=700), group=32), 2, 128),
    # g = 32 inside 64-column blocks; 2 bits
    ("dyn32_block64_2bit", dataclasses.replace(
        CONFIGS[5][1].scaled(130, 256, 2048, chunk=512), group=32, block=64), 4, 64),
    # g = 128 under blocks of 256 (the kernel still walks 128-column blocks); m >= 256 reaches
    # the pair tail GEMM
    ("dyn128_block256_pair_tail", dataclasses.replace(
        CONFIGS[2][0].scaled(300, 1100, 2500, chunk=1000), block=256), 10, 256),
]


@pytest.mark.parametrize("name,spec,seed,block", DYNAMIC, ids=[c[0] for c in DYNAMIC])
def test_dynamic_groups_parity(ctx, name, spec, seed, block):
    """grid_given = 2: each processing group's grid is fitted on the GPU from the current
    working weights at its start ([T] §8.3), against the oracle's dynamic recursion."""
    W, chunks = P.make_inputs(spec, seed)
    gpu = P.gpu_run(ctx, spec, W, chunks, block=block, grid_given=2)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, herr = P.check_hessian(gpu, Xt)
    res = P.check_layer(gpu, P.to_np64(W), H, spec, block=block, dynamic=True)
    print(name, f"H={herr:.2e}", {k: (f"{v:.2e}" if isinstance(v, float) else v) for k, v in res.items()})


def test_grid_modes_reject_unsupported(ctx):
    """Dynamic groups other than 32 / 128, or a group that a column block would split, the
    ternary grid with other than 2 bits, and unknown grid modes are argument errors reported by
    the library, not silently another grid."""
    import post_weight_quantization_17_b200 as G
    spec = CONFIGS[2][0].scaled(64, 256, 512, chunk=512)
    W, chunks = P.make_inputs(spec, 3)
    for group, block, mode, bits in ((64, 128, 2, 4), (128, 64, 2, 4), (32, 48, 2, 4),
                                     (8, 128, 4, 3), (8, 128, 4, 4), (128, 128, 5, 4),
                                     (128, 128, -1, 4)):
        bufs = G.LayerBuffers(64, 256, bits, group, W.device)
        bufs.R.copy_(torch.eye(256))
        with pytest.raises(RuntimeError):
            G.gptq_quantize_layer(ctx, W, bufs.R, None, bufs.dead, bits, group, block, mode,
                                  bufs.scales, bufs.zeros, bufs.codes, bufs.W_hat, bufs.col_loss)


@pytest.mark.parametrize("d", [700, 257, 1000])
def test_factor_stage_isolated(ctx, d):
    """Same fp32 H handed to both sides: R and H^-1 from the factorization alone (uneven
    recursion splits included)."""
    from oracle import gptq_oracle as O
    spec = CONFIGS[2][0].scaled(64, d, 4000, chunk=4000)
    W, chunks = P.make_inputs(spec, 11)
    H32 = O.hessian_tokens(torch.cat(chunks).cpu().double().numpy()).astype(np.float32)
    gpu = P.gpu_run(ctx, spec, W, chunks, H32=H32)
    o = O.prepare_with_retry(H32.astype(np.float64), spec.percdamp, False)
    Rg = gpu["R"].astype(np.float64)
    assert P.rel_fro(Rg, o["R"]) <= P.TOL_HINV
    assert P.rel_fro(Rg.T @ Rg, o["G"]) <= P.TOL_HINV
    assert abs(gpu["lam"] - o["lam"]) <= 1e-6 * o["lam"]


@pytest.mark.parametrize("block", [1, 7, 32, 128, 200])
def test_block_size_invariance(ctx, block):
    """Lazy blocks of any size give the unblocked result ([T] eq.(47)-(49))."""
    spec = CONFIGS[2][0].scaled(64, 260, 1200, chunk=600)
    W, chunks = P.make_inputs(spec, 21)
    gpu = P.gpu_run(ctx, spec, W, chunks, block=block)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, _ = P.check_hessian(gpu, Xt)
    P.check_layer(gpu, P.to_np64(W), H, spec, block=block)


def test_dead_features(ctx):
    spec = CONFIGS[3][0].scaled(48, 200, 800, chunk=400)
    W, chunks = P.make_inputs(spec, 31, zero_features=(0, 17, 130, 199))
    gpu = P.gpu_run(ctx, spec, W, chunks)
    assert gpu["dead"].nonzero()[0].tolist() == [0, 17, 130, 199]
    Xt = torch.cat(chunks).cpu().double().numpy()
    H, _ = P.check_hessian(gpu, Xt)
    P.check_layer(gpu, P.to_np64(W), H, spec)
    assert np.all(gpu["W_hat"][:, [0, 17, 130, 199]] == 0)


def test_unpack_roundtrip(ctx):
    import post_weight_quantization_17_b200 as G
    g = torch.Generator(device="cuda").manual_seed(5)
    for bits, d in [(2, 37), (3, 333), (4, 256), (8, 65)]:
        codes = torch.randint(0, 2 ** bits, (9, d), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
        packed = torch.empty(9, G.words_per_row(d, bits), dtype=torch.int32, device="cuda")
        G.gptq_pack(ctx, codes, bits, packed)
        back = torch.empty_like(codes)
        G.gptq_unpack(ctx, packed, d, bits, back)
        torch.cuda.synchronize()
        assert torch.equal(back, codes)


@pytest.mark.parametrize("d,n_tok,chunk", [(4096, 8192, 4096), (1000, 3001, 1024), (264, 130, 65)])
def test_hessian_tensor_path(ctx, d, n_tok, chunk):
    """The tensor-core Hessian over several waves of tiles, ragged d and token tails, and
    accumulation across chunks, against the fp64 oracle."""
    import post_weight_quantization_17_b200 as G
    from oracle import gptq_oracle as O
    spec = CONFIGS[2][0].scaled(64, d, n_tok, chunk=chunk)
    _, chunks = P.make_inputs(spec, 41)
    S = torch.empty(d, d, dtype=torch.float32, device="cuda")
    n = 0
    for c in chunks:
        n = G.gptq_hessian_accumulate(ctx, c, S, n)
    G.gptq_sync_status(ctx)
    Xt = torch.cat(chunks).cpu().double().numpy()
    H = O.hessian_tokens(Xt)
    Hg = np.tril(S.cpu().double().numpy()) * (2.0 / n)
    err = P.rel_fro(Hg, np.tril(H))
    print(f"d={d} N={n_tok} H rel err {err:.3e}")
    assert err <= P.TOL_H
