"""The C-ABI library loads and exports every symbol include/gptq.h declares; host-only logic
(argument checks that need no device, workspace sizing) behaves.  No GPU needed."""
import ctypes

import pytest

import post_weight_quantization_17_b200 as G


def test_every_header_symbol_is_exported():
    names = G.header_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(G._lib, n), f"{n} declared in include/gptq.h but not exported"


def test_binding_covers_header():
    declared = set(G.header_symbols())
    bound = set(G._SIGS)
    assert bound <= declared
    assert declared - bound == set(), f"unbound symbols: {declared - bound}"


def test_null_context_is_an_argument_error():
    L = G._lib
    n = ctypes.c_int64(0)
    assert L.gptq_hessian_accumulate(None, None, 0, 1, 1, None, ctypes.byref(n)) == G.GPTQ_ERR_ARG
    assert L.gptq_prepare_hinv(None, None, 0, 1, 0.01, 0, None, None, None, None, None) == G.GPTQ_ERR_ARG
    assert L.gptq_quantize_layer(None, None, 1, 1, 1, None, None, None, 4, -1, 128, 0, None, None,
                                 None, None, None) == G.GPTQ_ERR_ARG
    assert L.gptq_pack(None, None, 1, 1, 4, None) == G.GPTQ_ERR_ARG
    assert L.gptq_unpack(None, None, 1, 1, 4, None) == G.GPTQ_ERR_ARG
    assert L.gptq_dequant_matmul(None, None, 0, 1, 32, None, 1, 4, 128, None, 1, None, None,
                                 None) == G.GPTQ_ERR_ARG
    assert L.gptq_dequant_matmul_tiled(None, None, 0, 1, 32, None, 1, 128, 1, None, None,
                                       None) == G.GPTQ_ERR_ARG
    assert L.gptq_retile_codes(None, None, 1, 32, None) == G.GPTQ_ERR_ARG
    assert L.gptq_twosided_factor(None, None, 4) == G.GPTQ_ERR_ARG
    assert L.gptq_twosided_round(None, None, 2, 2, None, None, None, None) == G.GPTQ_ERR_ARG
    assert L.gptq_sync_status(None) == G.GPTQ_ERR_ARG
    assert L.gptq_set_wait_budget(None, 1) == G.GPTQ_ERR_ARG
    assert L.gptq_timing_enable(None, 1) == G.GPTQ_ERR_ARG
    assert L.gptq_timing_read(None, None, None) == G.GPTQ_ERR_ARG
    assert L.gptq_destroy(None) == G.GPTQ_ERR_ARG
    assert L.gptq_last_error(None) == b""


def test_create_rejects_bad_arguments():
    h = ctypes.c_void_p()
    assert G._lib.gptq_create(None, None, None, 1 << 20) == G.GPTQ_ERR_ARG
    assert G._lib.gptq_create(ctypes.byref(h), None, None, 16) == G.GPTQ_ERR_ARG


@pytest.mark.parametrize("m,d", [(64, 128), (4096, 4096), (4096, 11008), (12288, 49152)])
def test_workspace_bytes_cover_the_buffers(m, d):
    ws0 = G.gptq_workspace_bytes(m, d, False)
    ws1 = G.gptq_workspace_bytes(m, d, True)
    assert ws1 >= ws0 > 0
    # the factorization scratch alone is (d/2 + 64)^2 floats
    assert ws0 >= 4 * (d // 2 + 64) ** 2
    # act-order adds the permuted working copy (fp32) and permuted codes
    assert ws1 >= m * d * 5


def test_tiled_words():
    """16 KB (4096 words) per 128-row x 256-code tile, ragged blocks rounded up; 0 for empty."""
    assert G.gptq_tiled_words(128, 256) == 4096
    assert G.gptq_tiled_words(129, 256) == 2 * 4096
    assert G.gptq_tiled_words(12288, 49152) == 96 * 192 * 4096
    assert G.gptq_tiled_words(300, 1056) == 3 * 5 * 4096
    assert G.gptq_tiled_words(0, 256) == 0


def test_words_per_row():
    assert G.words_per_row(4096, 4) == 512
    assert G.words_per_row(11008, 3) == 1032
    assert G.words_per_row(37, 3) == 4
