"""Seeded synthetic layers shaped like the GPTQ workloads (weights W and calibration activations X).

This module holds no GPTQ arithmetic: it only draws random numbers and shapes them into the
inputs that both the CUDA path and the CPU oracle consume.  Every tensor is produced by a
``torch.Generator`` on the requested device, cast to the stated storage dtype, and is then
byte-identical for both consumers.

Recipes (the source pages measure on real LLM layers; these stand in for them):

* ``decay``         X = U diag(s) Z, U a random orthogonal matrix (QR of a Gaussian with a
                    sign-fixed diagonal), s geometric from 1 to 0.01, Z ~ N(0, 1).
* ``lowrank_t3``    X = diag(s) (F Y + 0.1 Xi), F ~ N(0, 1/r) of rank r, Y, Xi ~ N(0, 1),
                    s_i = |t_3| (per-feature Student-t scales: outlier features).
* ``swiglu``        X = SiLU(F G) * (F U), one mixing factor F ~ N(0, 1/r), G, U ~ N(0, 1).
* ``relu_lowrank``  X = ReLU(F Y + 0.1 Xi), F ~ N(0, 1/r).

X is produced token-major, one chunk ``[C, d]`` at a time (row t is token t's input vector),
which is the layout the Hessian accumulation consumes.  Chunk k of a layer with seed s draws
its token-dependent factors from seed ``s * 1000 + k + 1``, so any chunk can be regenerated on
its own; the feature-side factors (U, s, F) come from seed ``s * 1000``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator

import torch


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape and quantization settings of one synthetic linear layer."""

    name: str
    m: int                     # output features (rows of W)
    d: int                     # input features (columns of W, rows of X)
    n_tokens: int              # calibration tokens N
    bits: int
    group: int                 # -1 = one grid per row
    block: int
    act_order: bool
    percdamp: float = 0.01
    w_dtype: str = "f16"       # storage dtype of W: f16 | f32 | bf16
    x_dtype: str = "bf16"      # storage dtype of X: bf16 | f16 | f32
    w_std: float = 0.02
    outlier_frac: float = 0.0  # fraction of W columns scaled by outlier_scale
    outlier_scale: float = 1.0
    x_kind: str = "decay"
    x_rank: int = 256
    chunk: int = 8192          # tokens per X chunk

    @property
    def n_groups(self) -> int:
        return 1 if self.group == -1 else -(-self.d // self.group)

    @property
    def n_chunks(self) -> int:
        return -(-self.n_tokens // self.chunk)

    def chunk_rows(self, k: int) -> int:
        return min(self.chunk, self.n_tokens - k * self.chunk)

    def scaled(self, m: int, d: int, n_tokens: int, chunk: int | None = None, **kw) -> "LayerSpec":
        """Same recipe at another size (used for parity cases the oracle finishes in seconds)."""
        rank = min(self.x_rank, max(8, d // 4))
        return dataclasses.replace(self, m=m, d=d, n_tokens=n_tokens,
                                   chunk=chunk or min(self.chunk, n_tokens), x_rank=rank,
                                   name=f"{self.name}@{m}x{d}xN{n_tokens}", **kw)


_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _DT[name]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_weight(spec: LayerSpec, seed: int, device="cpu") -> torch.Tensor:
    """W [m, d]: N(0, w_std^2), with a fraction of whole columns scaled (outlier input features)."""
    g = _gen(device, seed * 1000 + 999_999)
    w = torch.randn(spec.m, spec.d, generator=g, device=device, dtype=torch.float32) * spec.w_std
    n_out = int(round(spec.outlier_frac * spec.d))
    if n_out > 0:
        cols = torch.randperm(spec.d, generator=g, device=device)[:n_out]
        w[:, cols] *= spec.outlier_scale
    return w.to(_DT[spec.w_dtype]).contiguous()


class XSource:
    """Token-major calibration activations of one layer, generated chunk by chunk."""

    def __init__(self, spec: LayerSpec, seed: int, device="cpu"):
        self.spec, self.seed, self.device = spec, seed, device
        g = _gen(device, seed * 1000)
        d, r = spec.d, spec.x_rank
        f32 = torch.float32
        self._feat = {}
        if spec.x_kind == "decay":
            a = torch.randn(d, d, generator=g, device=device, dtype=f32)
            q, rr = torch.linalg.qr(a)
            q = q * torch.sign(torch.diagonal(rr)).unsqueeze(0)
            s = torch.logspace(0.0, -2.0, d, device=device, dtype=f32)
            # token-major chunk = Z_c^T (U diag(s))^T
            self._feat["right"] = (q * s.unsqueeze(0)).t().contiguous()
        elif spec.x_kind in ("lowrank_t3", "relu_lowrank", "swiglu"):
            self._feat["F"] = torch.randn(d, r, generator=g, device=device, dtype=f32) / math.sqrt(r)
            if spec.x_kind == "lowrank_t3":
                # Student-t with 3 degrees of freedom: N(0,1) / sqrt(chi2_3 / 3)
                z = torch.randn(d, generator=g, device=device, dtype=f32)
                chi = (torch.randn(3, d, generator=g, device=device, dtype=f32) ** 2).sum(0)
                self._feat["s"] = (z / torch.sqrt(chi / 3.0)).abs()
        else:
            raise ValueError(spec.x_kind)

    def chunk(self, k: int) -> torch.Tensor:
        """Chunk k as a contiguous ``[C_k, d]`` tensor in the layer's X dtype."""
        spec = self.spec
        c = spec.chunk_rows(k)
        g = _gen(self.device, self.seed * 1000 + k + 1)
        f32 = torch.float32
        d, r = spec.d, spec.x_rank
        if spec.x_kind == "decay":
            z = torch.randn(c, d, generator=g, device=self.device, dtype=f32)
            x = z @ self._feat["right"]
        elif spec.x_kind == "lowrank_t3":
            y = torch.randn(c, r, generator=g, device=self.device, dtype=f32)
            xi = torch.randn(c, d, generator=g, device=self.device, dtype=f32)
            x = (y @ self._feat["F"].t() + 0.1 * xi) * self._feat["s"].unsqueeze(0)
        elif spec.x_kind == "relu_lowrank":
            y = torch.randn(c, r, generator=g, device=self.device, dtype=f32)
            xi = torch.randn(c, d, generator=g, device=self.device, dtype=f32)
            x = torch.relu(y @ self._feat["F"].t() + 0.1 * xi)
        else:  # swiglu
            gg = torch.randn(c, r, generator=g, device=self.device, dtype=f32)
            uu = torch.randn(c, r, generator=g, device=self.device, dtype=f32)
            ft = self._feat["F"].t()
            x = torch.nn.functional.silu(gg @ ft) * (uu @ ft)
        return x.to(_DT[spec.x_dtype]).contiguous()

    def chunks(self) -> Iterator[torch.Tensor]:
        for k in range(self.spec.n_chunks):
            yield self.chunk(k)

    def full(self) -> torch.Tensor:
        """All tokens as one ``[N, d]`` tensor."""
        return torch.cat(list(self.chunks()), dim=0)


# The five workloads: a tiny layer, a Llama-7B q_proj, an MLP down_proj with act-order,
# one 7B decoder block (7 matrices over 4 shared inputs), and a 175B-shaped fc2.
CONFIGS: dict[int, list[LayerSpec]] = {
    1: [LayerSpec("tiny_64x128", 64, 128, 256, bits=4, group=-1, block=32, act_order=False,
                  w_dtype="f32", x_dtype="f32", w_std=0.02, x_kind="decay", chunk=256)],
    2: [LayerSpec("q_proj_4096x4096", 4096, 4096, 262144, bits=4, group=128, block=128,
                  act_order=False, w_std=0.02, outlier_frac=0.01, outlier_scale=10.0,
                  x_kind="lowrank_t3", x_rank=256)],
    3: [LayerSpec("down_proj_4096x11008", 4096, 11008, 131072, bits=3, group=128, block=128,
                  act_order=True, w_std=0.015, x_kind="swiglu", x_rank=512)],
    4: [LayerSpec(f"{n}_{m}x{d}", m, d, 65536, bits=4, group=128, block=128, act_order=False,
                  w_std=0.02, x_kind="decay")
        for n, m, d in [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
                        ("o", 4096, 4096), ("gate", 11008, 4096), ("up", 11008, 4096),
                        ("down", 4096, 11008)]],
    5: [LayerSpec("fc2_12288x49152", 12288, 49152, 65536, bits=b, group=128, block=128,
                  act_order=False, w_std=0.01, outlier_frac=0.005, outlier_scale=8.0,
                  x_kind="relu_lowrank", x_rank=1024) for b in (4, 2)],
}

# Config 4: which matrices share one calibration input (one Hessian, one factorization).
BLOCK7B_SHARED_INPUT = {"qkv_in": ("q", "k", "v"), "o_in": ("o",),
                        "gateup_in": ("gate", "up"), "down_in": ("down",)}
