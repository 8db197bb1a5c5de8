"""Seeded synthetic GPTQ workloads shared by the tests, the benchmark and the oracle."""
from .synth import CONFIGS, BLOCK7B_SHARED_INPUT, LayerSpec, XSource, make_weight, torch_dtype  # noqa: F401
