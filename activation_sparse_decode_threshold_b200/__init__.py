"""Predictor-guided, neuron-aware sparse FFN decode for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libpi_ffn.so`` (``include/pi_ffn.h``),
built from ``csrc/`` by ``build.py``.  ``binding`` is a thin ctypes layer with
the same entry-point names; ``synth`` draws the seeded synthetic workloads.
"""
from . import binding  # noqa: F401  (loads the library lazily, fails loudly if absent)

__all__ = ["binding"]
