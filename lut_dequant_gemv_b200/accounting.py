"""Byte and bit accounting for one Dense-and-Sparse layer.

Storage per layer ("SqueezeLLM: Dense-and-Sparse Quantization", §3.4
"The 3/4-bit storage format" and "The Sparse Matrix Storage Format"):

* codes: exactly ``bits`` bits per weight, no padding            N*K*b/8 bytes
* LUT:   one table of 2**b fp16 centroids per output row          N*2**b*2 bytes
* CSR:   fp16 value + int32 column per nonzero, int32 row pointer 6*nnz + 4*(N+1)

The average-bit figure the pages print counts the codes, the LUTs and the
value+column of each nonzero (the row pointer is not part of it); the
algorithmic traffic of one GEMV call adds the row pointer and the fp16
activations read and outputs written.
"""
from __future__ import annotations

from typing import Iterable, Tuple


def code_bytes(n_out: int, k_in: int, bits: int) -> int:
    return n_out * k_in * bits // 8


def lut_bytes(n_out: int, bits: int) -> int:
    return n_out * (1 << bits) * 2


def csr_bytes(n_out: int, nnz: int, col_bytes: int = 4) -> int:
    """Value (fp16) + column per nonzero, plus the row pointer (int32)."""
    if nnz == 0:
        return 0
    return nnz * (2 + col_bytes) + 4 * (n_out + 1)


def gemv_bytes(n_out: int, k_in: int, bits: int, nnz: int, batch: int) -> int:
    """Algorithmic HBM bytes of one y = (Q + S) x call: every stored byte of
    the layer is read once, x is read once, y is written once."""
    return (code_bytes(n_out, k_in, bits) + lut_bytes(n_out, bits) + csr_bytes(n_out, nnz)
            + 2 * batch * (k_in + n_out))


def gemv_flops(n_out: int, k_in: int, nnz: int, batch: int) -> int:
    return 2 * batch * (n_out * k_in + nnz)


def fp16_dense_bytes(n_out: int, k_in: int, batch: int) -> int:
    """Bytes of the fp16 dense matrix-vector product used as a bandwidth yardstick."""
    return 2 * n_out * k_in + 2 * batch * (k_in + n_out)


def avg_bits(layers: Iterable[Tuple[int, int]], bits: int, density: float, bits_per_nnz: int = 48) -> float:
    """Average storage bits per weight over a set of (N, K) layers:
    codes + per-row LUTs + ``bits_per_nnz`` per outlier."""
    total_w = 0
    total_bits = 0.0
    for n, k in layers:
        total_w += n * k
        total_bits += n * k * bits + n * (1 << bits) * 16 + density * n * k * bits_per_nnz
    return total_bits / total_w


LLAMA7B_LAYER = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
