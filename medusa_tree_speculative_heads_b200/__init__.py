"""B200-native Medusa speculative decode step.

The computation lives in libmedusa.so (CUDA, sm_100a) behind the C ABI of
include/medusa.h; ``binding`` mirrors that ABI one to one and ``api`` adds
tensor-level conveniences.  ``inputs`` draws the seeded synthetic workloads.
"""
from . import binding  # noqa: F401  (loads nothing until the first call)
from .binding import MedusaError, Tree  # noqa: F401

__all__ = ["binding", "api", "inputs", "MedusaError", "Tree"]
