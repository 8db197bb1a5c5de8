"""CPU fp64 oracle for the GPTQ hot path (test infrastructure; see gptq_oracle.py)."""
from . import gptq_oracle  # noqa: F401
