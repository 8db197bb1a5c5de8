"""GPU parity of the W4A16 product Y = X Ŵᵀ over the packed codes (gptq_dequant_matmul) against
the oracle's dequantize-then-multiply, on seeded inputs.

Tolerance, from the arithmetic: Ŵ and X enter exactly (X is bf16/fp16/fp32, (c - z) is an exact
small integer, Δ is the stored fp32 scale), so the only error is fp32 accumulation of d
products plus the Δ scaling of each partial sum.  Recursive fp32 summation of d terms is within
γ_d = d u / (1 - d u) of Σ |x w| (u = 2^-24); the tensor core's internal adds are allowed twice
that, so every element must satisfy |Y - Y_oracle| <= 2 (d + 2) u Σ_k |X[t, k] Ŵ[r, k]|.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import gptq_oracle as O  # noqa: E402

U = 2.0 ** -24


@pytest.fixture(scope="module")
def ctx():
    import post_weight_quantization_17_b200 as G
    c = G.Context(m_max=4096, d_max=4096, act_order=True)
    yield c
    c.close()


def _inputs(T, m, d, bits, group, xdt, seed, ng=None):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** bits, size=(m, d))
    if ng is None:
        ng = 1 if group == -1 else -(-d // group)
    scales = rng.uniform(1e-3, 2e-2, (m, ng)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, (m, ng)).astype(np.int32)
    packed = O.pack(codes, bits).astype(np.uint32)
    X = torch.from_numpy(rng.normal(0, 1, (T, d)).astype(np.float32)).to(xdt)
    return codes, scales, zeros, packed, X


def _run(ctx, X, packed, d, bits, group, scales, zeros, group_id=None):
    import post_weight_quantization_17_b200 as G
    T, m = X.shape[0], packed.shape[0]
    Y = torch.full((T, m), float("nan"), dtype=torch.float32, device="cuda")
    gid = None if group_id is None else torch.from_numpy(np.asarray(group_id, np.int32)).cuda()
    G.gptq_dequant_matmul(ctx, X.cuda(), torch.from_numpy(packed.view(np.int32)).cuda(), d, bits,
                          group, torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(),
                          Y, group_id=gid)
    G.gptq_sync_status(ctx)
    torch.cuda.synchronize()
    return Y.cpu().numpy().astype(np.float64)


def _check(Y, X, packed, d, bits, scales, zeros, group, group_id=None):
    Xn = X.float().double().numpy()
    Yo = O.dequant_matmul(Xn, packed, d, bits, scales, zeros, group, group_id=group_id)
    codes = O.unpack(packed, d, bits)
    gid = (np.asarray(group_id) if group_id is not None else
           (np.zeros(d, np.int64) if group == -1 else np.arange(d) // group))
    W_abs = np.abs(scales[:, gid].astype(np.float64) * (codes - zeros[:, gid]))
    bound = 2 * (d + 2) * U * (np.abs(Xn) @ W_abs.T)
    err = np.abs(Y - Yo)
    assert np.all(np.isfinite(Y)), "unwritten or non-finite outputs"
    ratio = float(np.max(err / np.maximum(bound, 1e-300)))
    assert np.all(err <= bound), f"max error / bound = {ratio:.3f}"
    rel = float(np.linalg.norm(Y - Yo) / np.linalg.norm(Yo))
    return rel, ratio


CASES = [
    # (name, T, m, d, bits, group, x dtype) -- the first four take the tensor-core path
    ("decode_T1_qproj_bf16", 1, 4096, 4096, 4, 128, torch.bfloat16),
    ("decode_T16_fp16", 16, 1024, 2048, 4, 128, torch.float16),
    ("T48_ragged_rows_and_tail", 48, 300, 1056, 4, 128, torch.bfloat16),
    ("T200_rowgrid", 200, 256, 512, 4, -1, torch.bfloat16),
    ("T130_g256_fp16", 130, 384, 768, 4, 256, torch.float16),
    # CUDA-core path: other widths, groups, fp32 X, ragged d
    ("simt_3bit_g32_fp32", 5, 200, 333, 3, 32, torch.float32),
    ("simt_4bit_g64", 9, 130, 640, 4, 64, torch.bfloat16),
    ("simt_2bit_ternary_like_g8", 3, 64, 256, 2, 8, torch.float16),
    ("simt_8bit_row", 2, 33, 100, 8, -1, torch.float32),
]


@pytest.mark.parametrize("k", range(len(CASES)), ids=[c[0] for c in CASES])
def test_dequant_matmul_parity(ctx, k):
    name, T, m, d, bits, group, xdt = CASES[k]
    _, scales, zeros, packed, X = _inputs(T, m, d, bits, group, xdt, 100 + k)
    Y = _run(ctx, X, packed, d, bits, group, scales, zeros)
    rel, ratio = _check(Y, X, packed, d, bits, scales, zeros, group)
    print(name, f"rel={rel:.2e} max_err/bound={ratio:.2e}")


def test_dequant_matmul_group_id(ctx):
    """Per-column grid indices (dynamic groups under act-order: group_id[π_j] = j / g)."""
    T, m, d, bits, g = 7, 96, 384, 4, 32
    perm = np.random.default_rng(5).permutation(d)
    gid = np.empty(d, np.int64)
    gid[perm] = np.arange(d) // g
    _, scales, zeros, packed, X = _inputs(T, m, d, bits, g, torch.bfloat16, 6, ng=d // g)
    Y = _run(ctx, X, packed, d, bits, g, scales, zeros, group_id=gid)
    rel, ratio = _check(Y, X, packed, d, bits, scales, zeros, g, group_id=gid)
    print("group_id", f"rel={rel:.2e} max_err/bound={ratio:.2e}")


def test_dequant_matmul_layer_roundtrip(ctx):
    """End to end: a layer quantized by the library, packed by the library, multiplied by the
    library, against X Ŵᵀ for the Ŵ the library returned (the oracle pins that Ŵ elsewhere)."""
    import post_weight_quantization_17_b200 as G
    from tests import _parity as P
    from workloads.synth import CONFIGS
    spec = CONFIGS[2][0].scaled(256, 512, 2048, chunk=1024)
    W, chunks = P.make_inputs(spec, 7)
    gpu = P.gpu_run(ctx, spec, W, chunks)
    X = torch.randn(24, 512, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    Y = _run(ctx, X, gpu["packed"].view(np.uint32), 512, 4, 128, gpu["scales"], gpu["zeros"])
    Xn = X.float().double().numpy()
    ref = Xn @ gpu["W_hat"].astype(np.float64).T
    bound = 2 * 514 * U * (np.abs(Xn) @ np.abs(gpu["W_hat"].astype(np.float64)).T)
    assert np.all(np.abs(Y - ref) <= bound)


@pytest.mark.parametrize("T", [1, 16])
def test_dequant_matmul_fc2_full_size_sampled(ctx, T):
    """The 175B fc2 shape at full size (12288 x 49152, 4-bit g128, 302 MB of codes): random
    packed words are valid codes; 48 sampled rows are checked against the oracle."""
    import post_weight_quantization_17_b200 as G
    m, d, g = 12288, 49152, 128
    gen = torch.Generator(device="cuda").manual_seed(9)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (m, d // 8), dtype=torch.int32, device="cuda",
                           generator=gen)
    scales = torch.rand(m, d // g, device="cuda", generator=gen) * 0.02 + 1e-3
    zeros = torch.randint(0, 16, (m, d // g), dtype=torch.int32, device="cuda", generator=gen)
    X = torch.randn(T, d, device="cuda", generator=gen).to(torch.bfloat16)
    Y = torch.empty(T, m, dtype=torch.float32, device="cuda")
    G.gptq_dequant_matmul(ctx, X, packed, d, 4, g, scales, zeros, Y)
    G.gptq_sync_status(ctx)
    rows = np.random.default_rng(10).choice(m, 48, replace=False)
    pk = packed[rows].cpu().numpy().view(np.uint32)
    sc, ze = scales[rows].cpu().numpy(), zeros[rows].cpu().numpy()
    Yg = Y[:, rows].cpu().numpy().astype(np.float64)
    _check(Yg, X.cpu(), pk, d, 4, sc, ze, g)


@pytest.mark.xfail(strict=False, reason=(
    "open defect: the row-layout product is intermittently wrong on a band of rows at the full "
    "fc2 shape, while the tile-contiguous layout agrees with the oracle there"))
@pytest.mark.parametrize("T", [1, 16])
def test_dequant_matmul_fc2_every_row_row_layout_vs_tiled(ctx, T):
    """Every row of the full-size fc2 product (12288 x 49152, 4-bit g128) from the row layout
    against the same product from the tile-contiguous layout.  Both run the same kernel; only the
    codes' copies into shared memory differ, so the two agree to rounding (a differing split of K
    would change only the order of fp32 adds)."""
    import post_weight_quantization_17_b200 as G
    m, d, g = 12288, 49152, 128
    gen = torch.Generator(device="cuda").manual_seed(11)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (m, d // 8), dtype=torch.int32, device="cuda",
                           generator=gen)
    scales = torch.rand(m, d // g, device="cuda", generator=gen) * 0.02 + 1e-3
    zeros = torch.randint(0, 16, (m, d // g), dtype=torch.int32, device="cuda", generator=gen)
    X = torch.randn(T, d, device="cuda", generator=gen).to(torch.bfloat16)
    tiled = torch.zeros(G.gptq_tiled_words(m, d), dtype=torch.int32, device="cuda")
    G.gptq_retile_codes(ctx, packed, d, tiled)
    Yr = torch.empty(T, m, dtype=torch.float32, device="cuda")
    Yt = torch.empty(T, m, dtype=torch.float32, device="cuda")
    G.gptq_dequant_matmul(ctx, X, packed, d, 4, g, scales, zeros, Yr)
    G.gptq_dequant_matmul_tiled(ctx, X, tiled, m, g, scales, zeros, Yt)
    G.gptq_sync_status(ctx)
    rms = float(Yt.square().mean().sqrt())
    worst = float((Yr - Yt).abs().max()) / rms
    assert worst <= 1e-4, f"max |row layout - tiled| / rms = {worst:.2e}"
