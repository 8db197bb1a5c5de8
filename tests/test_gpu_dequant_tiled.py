"""GPU parity of the tile-contiguous codes path: the re-layout bit-exact against the oracle's
definition, and the product over it against the oracle's dequantize-then-multiply."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from oracle import gptq_oracle as O  # noqa: E402
from tests.test_gpu_dequant import U, _check, _inputs  # noqa: E402


@pytest.fixture(scope="module")
def ctx():
    import post_weight_quantization_17_b200 as G
    c = G.Context(m_max=4096, d_max=4096, act_order=True)
    yield c
    c.close()


@pytest.mark.parametrize("m,d", [(300, 1056), (128, 256), (4096, 4096), (77, 96)])
def test_retile_bit_exact(ctx, m, d):
    import post_weight_quantization_17_b200 as G
    rng = np.random.default_rng(m + d)
    packed = rng.integers(0, 2 ** 32, size=(m, d // 8), dtype=np.uint64).astype(np.uint32)
    tiled = torch.zeros(G.gptq_tiled_words(m, d), dtype=torch.int32, device="cuda")
    G.gptq_retile_codes(ctx, torch.from_numpy(packed.view(np.int32)).cuda(), d, tiled)
    torch.cuda.synchronize()
    assert np.array_equal(tiled.cpu().numpy().view(np.uint32), O.tile_codes4(packed, m, d))


CASES = [(1, 4096, 4096, 128, torch.bfloat16), (16, 1024, 2048, 128, torch.float16),
         (48, 300, 1056, 128, torch.bfloat16), (200, 256, 512, -1, torch.bfloat16),
         (130, 384, 768, 256, torch.float16)]


@pytest.mark.parametrize("k", range(len(CASES)))
def test_dequant_matmul_tiled_parity(ctx, k):
    import post_weight_quantization_17_b200 as G
    T, m, d, group, xdt = CASES[k]
    _, scales, zeros, packed, X = _inputs(T, m, d, 4, group, xdt, 200 + k)
    tiled = torch.zeros(G.gptq_tiled_words(m, d), dtype=torch.int32, device="cuda")
    G.gptq_retile_codes(ctx, torch.from_numpy(packed.view(np.int32)).cuda(), d, tiled)
    Y = torch.full((T, m), float("nan"), device="cuda")
    G.gptq_dequant_matmul_tiled(ctx, X.cuda(), tiled, m, group, torch.from_numpy(scales).cuda(),
                                torch.from_numpy(zeros).cuda(), Y)
    G.gptq_sync_status(ctx)
    rel, ratio = _check(Y.cpu().numpy().astype(np.float64), X, packed, d, 4, scales, zeros, group)
    print(CASES[k][:4], f"rel={rel:.2e} max_err/bound={ratio:.2e}")
