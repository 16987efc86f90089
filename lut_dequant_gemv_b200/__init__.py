"""Dense-and-Sparse LUT-dequant GEMV for NVIDIA B200 (sm_100a).

y = (Q + S) x, where Q holds 3/4-bit codes into per-output-row fp16 lookup
tables and S is an fp16 CSR outlier matrix ("SqueezeLLM: Dense-and-Sparse
Quantization", §3.4 "Kernel Implementation").

The compute path is the CUDA library ``libsqz.so`` (C ABI declared in
``include/sqz.h``); :mod:`lut_dequant_gemv_b200.binding` marshals arguments
to it.  The binding is imported lazily so that host-only utilities
(:mod:`lut_dequant_gemv_b200.accounting`) work on machines without the
built library; every compute call fails loudly if the library is missing.
"""
from __future__ import annotations

import importlib

__all__ = ["binding", "accounting"]


def __getattr__(name):
    if name in ("binding", "accounting"):
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
