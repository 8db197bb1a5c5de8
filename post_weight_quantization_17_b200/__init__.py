"""Python binding of libgptq_b200.so (the C ABI declared in include/gptq.h).

Argument marshalling only: every step of the GPTQ path runs in the library's sm_100a kernels.
PyTorch provides device memory and streams.  Importing this module loads the library and
raises if it is missing or lacks a symbol: there is no fallback path.

The functions carry the C names; tensors are passed as device pointers, scalars by value.
`quantize_layer_pipeline` strings the four hot-path calls together for one layer.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "gptq.h")

GPTQ_OK, GPTQ_ERR_ARG, GPTQ_ERR_CUDA, GPTQ_ERR_NOT_PD, GPTQ_ERR_NONFINITE, \
    GPTQ_ERR_TIMEOUT, GPTQ_ERR_NOMEM = range(7)
GPTQ_BF16, GPTQ_F16, GPTQ_F32 = 0, 1, 2
STATUS_NAMES = {0: "OK", 1: "ERR_ARG", 2: "ERR_CUDA", 3: "ERR_NOT_PD", 4: "ERR_NONFINITE",
                5: "ERR_TIMEOUT", 6: "ERR_NOMEM"}

_DTYPE_CODE = {torch.bfloat16: GPTQ_BF16, torch.float16: GPTQ_F16, torch.float32: GPTQ_F32}

# stages of gptq_timing_read, in the order of the GPTQ_STAGE_* constants
STAGES = ("hessian", "prepare", "factor_base", "factor_gemm", "factor_copy", "grid", "column",
          "update", "output", "pack", "dequant", "twosided", "other")


class GPTQError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python post_weight_quantization_17_b200/build.py` (no fallback exists)")
_lib = ctypes.CDLL(LIB_PATH)

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "gptq_workspace_bytes": (_sz, [_i64, _i64, _i32]),
    "gptq_create": (_i32, [ctypes.POINTER(_vp), _vp, _vp, _sz]),
    "gptq_destroy": (_i32, [_vp]),
    "gptq_last_error": (ctypes.c_char_p, [_vp]),
    "gptq_kernel_launches": (ctypes.c_uint64, [_vp]),
    "gptq_sync_status": (_i32, [_vp]),
    "gptq_set_wait_budget": (_i32, [_vp, _i64]),
    "gptq_timing_enable": (_i32, [_vp, _i32]),
    "gptq_timing_read": (_i32, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)]),
    "gptq_hessian_accumulate": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, ctypes.POINTER(_i64)]),
    "gptq_prepare_hinv": (_i32, [_vp, _vp, _i64, _i64, ctypes.c_float, _i32, _vp, _vp, _vp,
                                 ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_i32)]),
    "gptq_quantize_layer": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _i32, _i32, _i32,
                                   _i32, _vp, _vp, _vp, _vp, _vp]),
    "gptq_quantize_layer_noalloc": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _i32, _i32,
                                           _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "gptq_pack": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp]),
    "gptq_unpack": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp]),
    "gptq_dequant_matmul": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _i64, _i32, _i32, _vp, _i64,
                                   _vp, _vp, _vp]),
    "gptq_tiled_words": (ctypes.c_longlong, [_i64, _i64]),
    "gptq_retile_codes": (_i32, [_vp, _vp, _i64, _i64, _vp]),
    "gptq_dequant_matmul_tiled": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _i64, _i32, _i64, _vp,
                                         _vp, _vp]),
    "gptq_twosided_factor": (_i32, [_vp, _vp, _i64]),
    "gptq_twosided_round": (_i32, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)  # AttributeError here means the library lacks a declared symbol
    _f.restype, _f.argtypes = _res, _args


def header_symbols(path: str = HEADER_PATH) -> list[str]:
    """Names of the functions declared in include/gptq.h."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_]+)\s*\(", text)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, dtype=None, name="tensor"):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


class Context:
    """A library context: the CUDA stream the calls are enqueued on and a device workspace
    (a torch uint8 tensor) sized for layers up to (m_max, d_max)."""

    def __init__(self, m_max: int, d_max: int, act_order: bool = True, stream=None,
                 device=None):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        nbytes = int(_lib.gptq_workspace_bytes(m_max, d_max, 1 if act_order else 0))
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            rc = _lib.gptq_create(ctypes.byref(h), ctypes.c_void_p(self.stream.cuda_stream),
                                  _ptr(self.workspace), nbytes)
        if rc != GPTQ_OK:
            raise GPTQError(rc, "gptq_create failed")
        self.handle = h

    def check(self, rc: int, what: str):
        if rc != GPTQ_OK:
            msg = _lib.gptq_last_error(self.handle) or b""
            raise GPTQError(rc, f"{what}: {msg.decode(errors='replace')}")

    def close(self):
        if getattr(self, "handle", None):
            _lib.gptq_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gptq_workspace_bytes(m: int, d: int, act_order: bool) -> int:
    return int(_lib.gptq_workspace_bytes(m, d, 1 if act_order else 0))


def gptq_kernel_launches(ctx: Context) -> int:
    return int(_lib.gptq_kernel_launches(ctx.handle))


def gptq_set_wait_budget(ctx: Context, cycles: int):
    """Wait budget of this context's pipelined kernels in GPU cycles (0 = the default)."""
    ctx.check(_lib.gptq_set_wait_budget(ctx.handle, int(cycles)), "gptq_set_wait_budget")


def gptq_timing_enable(ctx: Context, on: bool = True):
    """Time every launch of this context with CUDA events (serializes neighbouring launches)."""
    ctx.check(_lib.gptq_timing_enable(ctx.handle, 1 if on else 0), "gptq_timing_enable")


def gptq_timing_read(ctx: Context) -> dict:
    """{stage: (milliseconds summed over its timed launches, launches)} since the last read."""
    ms = (ctypes.c_double * len(STAGES))()
    n = (_i64 * len(STAGES))()
    ctx.check(_lib.gptq_timing_read(ctx.handle, ms, n), "gptq_timing_read")
    return {name: (ms[k], int(n[k])) for k, name in enumerate(STAGES) if n[k]}


def gptq_sync_status(ctx: Context) -> int:
    rc = _lib.gptq_sync_status(ctx.handle)
    ctx.check(rc, "gptq_sync_status")
    return rc


def gptq_hessian_accumulate(ctx: Context, Xc: torch.Tensor, S: torch.Tensor, n_total: int) -> int:
    """S (+)= Xc^T Xc for a token-major chunk Xc [n, d]; returns the new token count."""
    _dev(Xc, name="Xc")
    _dev(S, torch.float32, "S")
    n = ctypes.c_int64(n_total)
    rc = _lib.gptq_hessian_accumulate(ctx.handle, _ptr(Xc), _DTYPE_CODE[Xc.dtype], Xc.shape[0],
                                      Xc.shape[1], _ptr(S), ctypes.byref(n))
    ctx.check(rc, "gptq_hessian_accumulate")
    return n.value


def gptq_prepare_hinv(ctx: Context, S, n_total: int, percdamp: float, act_order: bool, R, perm,
                      dead):
    """Returns (damp_used, retries); R, perm, dead are written in place."""
    d = S.shape[0]
    for t, dt, nm in ((S, torch.float32, "S"), (R, torch.float32, "R"),
                      (perm, torch.int32, "perm"), (dead, torch.uint8, "dead")):
        _dev(t, dt, nm)
    lam = ctypes.c_float(0.0)
    retries = ctypes.c_int(0)
    rc = _lib.gptq_prepare_hinv(ctx.handle, _ptr(S), n_total, d, ctypes.c_float(percdamp),
                                1 if act_order else 0, _ptr(R), _ptr(perm), _ptr(dead),
                                ctypes.byref(lam), ctypes.byref(retries))
    ctx.check(rc, "gptq_prepare_hinv")
    return lam.value, retries.value


def gptq_quantize_layer(ctx: Context, W, R, perm, dead, bits: int, group: int, block: int,
                        grid_given, scales, zeros, codes, W_hat, col_loss):
    """perm / dead may be None (identity order / no dead features).  grid_given: False / 0 fit a
    static min-max grid, True / 1 use the given one, 2 dynamic groups, 3 fit a static symmetric
    grid, 4 fit the static ternary grid (bits = 2); see include/gptq.h."""
    m, d = W.shape
    _dev(W, name="W")
    for t, dt, nm in ((R, torch.float32, "R"), (scales, torch.float32, "scales"),
                      (zeros, torch.int32, "zeros"), (codes, torch.uint8, "codes"),
                      (W_hat, torch.float32, "W_hat"), (col_loss, torch.float32, "col_loss")):
        _dev(t, dt, nm)
    rc = _lib.gptq_quantize_layer(ctx.handle, _ptr(W), _DTYPE_CODE[W.dtype], m, d, _ptr(R),
                                  _ptr(perm), _ptr(dead), bits, group, block,
                                  int(grid_given), _ptr(scales), _ptr(zeros), _ptr(codes),
                                  _ptr(W_hat), _ptr(col_loss))
    ctx.check(rc, "gptq_quantize_layer")


def gptq_quantize_layer_noalloc(W, R, perm, dead, bits: int, group: int, block: int,
                                grid_given: bool, scales, zeros, codes, W_hat, col_loss,
                                stream=None) -> int:
    """gptq_quantize_layer without a context or workspace (fixed device scratch inside the
    library); synchronizes the stream and returns the status code (0 = OK)."""
    m, d = W.shape
    _dev(W, name="W")
    s = stream if stream is not None else torch.cuda.current_stream(W.device)
    with torch.cuda.device(W.device):   # the library resolves its scratch on the current device
        return int(_lib.gptq_quantize_layer_noalloc(
            ctypes.c_void_p(s.cuda_stream), _ptr(W), _DTYPE_CODE[W.dtype], m, d, _ptr(R),
            _ptr(perm), _ptr(dead), bits, group, block, int(grid_given), _ptr(scales),
            _ptr(zeros), _ptr(codes), _ptr(W_hat), _ptr(col_loss)))


def gptq_pack(ctx: Context, codes, bits: int, packed):
    m, d = codes.shape
    _dev(codes, torch.uint8, "codes")
    _dev(packed, torch.int32, "packed")
    rc = _lib.gptq_pack(ctx.handle, _ptr(codes), m, d, bits, _ptr(packed))
    ctx.check(rc, "gptq_pack")


def gptq_unpack(ctx: Context, packed, d: int, bits: int, codes):
    m = packed.shape[0]
    _dev(codes, torch.uint8, "codes")
    _dev(packed, torch.int32, "packed")
    rc = _lib.gptq_unpack(ctx.handle, _ptr(packed), m, d, bits, _ptr(codes))
    ctx.check(rc, "gptq_unpack")


def gptq_dequant_matmul(ctx: Context, X, packed, d: int, bits: int, group: int, scales, zeros,
                        Y, group_id=None):
    """Y [T, m] = X [T, d] Ŵᵀ from the packed codes (the W4A16 product; see include/gptq.h).
    group_id: per-column grid index [d] int32 (dynamic groups under act-order) or None."""
    T = X.shape[0]
    m = packed.shape[0]
    _dev(X, name="X")
    for t, dt, nm in ((packed, torch.int32, "packed"), (scales, torch.float32, "scales"),
                      (zeros, torch.int32, "zeros"), (Y, torch.float32, "Y")):
        _dev(t, dt, nm)
    if group_id is not None:
        _dev(group_id, torch.int32, "group_id")
    rc = _lib.gptq_dequant_matmul(ctx.handle, _ptr(X), _DTYPE_CODE[X.dtype], T, d, _ptr(packed),
                                  m, bits, group, _ptr(group_id), scales.shape[1], _ptr(scales),
                                  _ptr(zeros), _ptr(Y))
    ctx.check(rc, "gptq_dequant_matmul")


def gptq_tiled_words(m: int, d: int) -> int:
    return int(_lib.gptq_tiled_words(m, d))


def gptq_retile_codes(ctx: Context, packed, d: int, tiled):
    """4-bit packed codes [m, d / 8] -> the tile-contiguous copy (see include/gptq.h)."""
    _dev(packed, torch.int32, "packed")
    _dev(tiled, torch.int32, "tiled")
    ctx.check(_lib.gptq_retile_codes(ctx.handle, _ptr(packed), packed.shape[0], d, _ptr(tiled)),
              "gptq_retile_codes")


def gptq_dequant_matmul_tiled(ctx: Context, X, tiled, m: int, group: int, scales, zeros, Y):
    """Y [T, m] = X [T, d] Ŵᵀ over the tile-contiguous 4-bit codes."""
    T, d = X.shape
    _dev(X, name="X")
    for t, dt, nm in ((tiled, torch.int32, "tiled"), (scales, torch.float32, "scales"),
                      (zeros, torch.int32, "zeros"), (Y, torch.float32, "Y")):
        _dev(t, dt, nm)
    ctx.check(_lib.gptq_dequant_matmul_tiled(ctx.handle, _ptr(X), _DTYPE_CODE[X.dtype], T, d,
                                             _ptr(tiled), m, group, scales.shape[1],
                                             _ptr(scales), _ptr(zeros), _ptr(Y)),
              "gptq_dequant_matmul_tiled")


def gptq_twosided_factor(ctx: Context, G):
    """In place: G [k, k] fp32 (symmetric positive definite) -> R upper with R^T R = G^-1."""
    _dev(G, torch.float32, "G")
    ctx.check(_lib.gptq_twosided_factor(ctx.handle, _ptr(G), G.shape[0]), "gptq_twosided_factor")


def gptq_twosided_round(ctx: Context, X, RA, RB, Z, eta):
    """Two-sided GPTQ rounding of X [m, n] with the factors from gptq_twosided_factor; writes the
    integers Z and the scaled residuals eta (see include/gptq.h)."""
    m, n = X.shape
    for t, nm in ((X, "X"), (RA, "RA"), (RB, "RB"), (Z, "Z"), (eta, "eta")):
        _dev(t, torch.float32, nm)
    ctx.check(_lib.gptq_twosided_round(ctx.handle, _ptr(X), m, n, _ptr(RA), _ptr(RB), _ptr(Z),
                                       _ptr(eta)), "gptq_twosided_round")


def words_per_row(d: int, bits: int) -> int:
    return -(-(d * bits) // 32)


class LayerBuffers:
    """Device buffers of one layer's outputs (allocated once, reused across calls).  With
    with_factor=False only the quantization outputs are allocated (for matrices that share
    another layer's S, R, perm and dead)."""

    def __init__(self, m: int, d: int, bits: int, group: int, device, with_factor: bool = True):
        ng = 1 if group == -1 else -(-d // group)
        f32 = torch.float32
        if with_factor:
            self.S = torch.empty(d, d, dtype=f32, device=device)
            self.R = torch.empty(d, d, dtype=f32, device=device)
            self.perm = torch.empty(d, dtype=torch.int32, device=device)
            self.dead = torch.empty(d, dtype=torch.uint8, device=device)
        self.scales = torch.empty(m, ng, dtype=f32, device=device)
        self.zeros = torch.empty(m, ng, dtype=torch.int32, device=device)
        self.codes = torch.empty(m, d, dtype=torch.uint8, device=device)
        self.W_hat = torch.empty(m, d, dtype=f32, device=device)
        self.col_loss = torch.empty(d, dtype=f32, device=device)
        self.packed = torch.empty(m, words_per_row(d, bits), dtype=torch.int32, device=device)


def quantize_layer_pipeline(ctx: Context, X_chunks, W, bits: int, group: int, block: int,
                            percdamp: float = 0.01, act_order: bool = False,
                            bufs: LayerBuffers | None = None, H=None):
    """One layer through the four C-ABI calls: accumulate S over the token chunks (or take a
    normalised H), prepare R, quantize, pack.  Returns the LayerBuffers plus (damp, retries)."""
    m, d = W.shape
    if bufs is None:
        bufs = LayerBuffers(m, d, bits, group, W.device)
    if H is None:
        n_total = 0
        for xc in X_chunks:
            n_total = gptq_hessian_accumulate(ctx, xc, bufs.S, n_total)
    else:
        bufs.S.copy_(H)
        n_total = 0
    lam, retries = gptq_prepare_hinv(ctx, bufs.S, n_total, percdamp, act_order, bufs.R, bufs.perm,
                                     bufs.dead)
    gptq_quantize_layer(ctx, W, bufs.R, bufs.perm if act_order else None, bufs.dead, bits, group,
                        block, False, bufs.scales, bufs.zeros, bufs.codes, bufs.W_hat,
                        bufs.col_loss)
    gptq_pack(ctx, bufs.codes, bits, bufs.packed)
    return bufs, lam, retries
