"""CPU oracle for the Dense-and-Sparse quantized GEMV (fp64).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only users.  The product (the CUDA
library and its Python binding) never imports this package.

The arithmetic lives in plain C (``sqz_oracle.c``); this module compiles it
with gcc and marshals numpy arrays.  See the C file's header for the
definition it follows ("SqueezeLLM: Dense-and-Sparse Quantization", §3.4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sqz_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (strict IEEE: no contraction, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, c_int = ctypes.c_int32, ctypes.c_int64, ctypes.c_int
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_words_per_row.argtypes = [i64, c_int]
    lib.oracle_words_per_row.restype = i64
    lib.oracle_code.argtypes = [P, c_int, i64]
    lib.oracle_code.restype = ctypes.c_uint32
    lib.oracle_unpack.argtypes = [i32, i32, c_int, P, P]
    lib.oracle_unpack.restype = c_int
    lib.oracle_pack.argtypes = [i32, i32, c_int, P, P]
    lib.oracle_pack.restype = c_int
    lib.oracle_dequant.argtypes = [i32, i32, c_int, P, P, P]
    lib.oracle_dequant.restype = c_int
    lib.oracle_check_csr.argtypes = [i32, i32, i64, P, P]
    lib.oracle_check_csr.restype = c_int
    lib.oracle_gemv.argtypes = [i32, i32, c_int, P, P, i64, P, P, P, P, i32, i64, P, i64, P, P]
    lib.oracle_gemv.restype = c_int
    lib.oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_outliers_per_tail.argtypes = [i64, ctypes.c_double]
    lib.oracle_outliers_per_tail.restype = i64
    lib.oracle_select_outliers.argtypes = [i32, i32, P, i64, P]
    lib.oracle_select_outliers.restype = c_int
    lib.oracle_kmeans_row.argtypes = [i64, P, c_int, c_int, P]
    lib.oracle_kmeans_row.restype = c_int
    lib.oracle_encode.argtypes = [i32, i32, c_int, P, ctypes.c_double, c_int, P, i32, P, P, P, P, P, i64, P, P]
    lib.oracle_encode.restype = c_int
    return lib


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """Thin marshalling layer over one loaded copy of the C oracle."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def half_to_double(self, h: int) -> float:
        return float(self.lib.oracle_half_to_double(int(h)))

    def unpack(self, codes: np.ndarray, n_out: int, k_in: int, bits: int) -> np.ndarray:
        codes = _c(codes, np.uint32)
        out = np.empty((n_out, k_in), dtype=np.uint8)
        rc = self.lib.oracle_unpack(n_out, k_in, bits, _ptr(codes), _ptr(out))
        if rc:
            raise ValueError("oracle_unpack: bad arguments")
        return out

    def pack(self, code_matrix: np.ndarray, bits: int) -> np.ndarray:
        cm = _c(code_matrix, np.uint8)
        n_out, k_in = cm.shape
        wpr = self.lib.oracle_words_per_row(k_in, bits)
        if wpr < 0:
            raise ValueError("K*bits must be a multiple of 32")
        out = np.empty((n_out, wpr), dtype=np.uint32)
        rc = self.lib.oracle_pack(n_out, k_in, bits, _ptr(cm), _ptr(out))
        if rc:
            raise ValueError("oracle_pack: bad arguments")
        return out

    def dequant(self, codes, lut, n_out: int, k_in: int, bits: int) -> np.ndarray:
        codes, lut = _c(codes, np.uint32), _c(lut, np.uint16)
        out = np.empty((n_out, k_in), dtype=np.uint16)
        rc = self.lib.oracle_dequant(n_out, k_in, bits, _ptr(codes), _ptr(lut), _ptr(out))
        if rc:
            raise ValueError("oracle_dequant: bad arguments")
        return out

    def check_csr(self, n_out: int, k_in: int, rowptr, col) -> bool:
        rowptr, col = _c(rowptr, np.int32), _c(col, np.int32)
        nnz = 0 if col is None else int(col.shape[0])
        return self.lib.oracle_check_csr(n_out, k_in, nnz, _ptr(rowptr), _ptr(col)) == 0

    def gemv(self, n_out: int, k_in: int, bits: int, codes, lut, rowptr, col, val, x,
             rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
        """Return (y, bound), each float64 [batch, n_rows]."""
        codes, lut = _c(codes, np.uint32), _c(lut, np.uint16)
        rowptr, col, val = _c(rowptr, np.int32), _c(col, np.int32), _c(val, np.uint16)
        x = _c(x, np.uint16)
        if x.ndim == 1:
            x = x[None, :]
        batch, ldx = x.shape
        nnz = 0 if col is None else int(col.shape[0])
        rows_c = None if rows is None else _c(rows, np.int32)
        n_rows = n_out if rows_c is None else int(rows_c.shape[0])
        y = np.empty((batch, n_rows), dtype=np.float64)
        bound = np.empty((batch, n_rows), dtype=np.float64)
        rc = self.lib.oracle_gemv(n_out, k_in, bits, _ptr(codes), _ptr(lut), nnz, _ptr(rowptr), _ptr(col),
                                  _ptr(val), _ptr(x), batch, ldx, _ptr(rows_c), n_rows, _ptr(y), _ptr(bound))
        if rc:
            raise ValueError("oracle_gemv: bad arguments")
        return y, bound

    # ---- encoder (Dense-and-Sparse split + per-row 1-D k-means), fp64
    def double_to_half(self, v: float) -> int:
        return int(self.lib.oracle_double_to_half(float(v)))

    def outliers_per_tail(self, n: int, fraction: float) -> int:
        return int(self.lib.oracle_outliers_per_tail(int(n), float(fraction)))

    def select_outliers(self, w: np.ndarray, m: int) -> np.ndarray:
        """uint8 marks [n_out, k_in]: 1 for the first m and last m weights in
        ascending (value, row-major position) order."""
        w = _c(w, np.uint16)
        n_out, k_in = w.shape
        marks = np.empty((n_out, k_in), dtype=np.uint8)
        if self.lib.oracle_select_outliers(n_out, k_in, _ptr(w), int(m), _ptr(marks)):
            raise ValueError("oracle_select_outliers: bad arguments")
        return marks

    def kmeans_row(self, d: np.ndarray, k: int, max_iters: int) -> Tuple[np.ndarray, int]:
        """(centroids float64 [k], iterations run) of 1-D Lloyd k-means."""
        d = _c(d, np.float64)
        c = np.empty(k, dtype=np.float64)
        it = self.lib.oracle_kmeans_row(int(d.shape[0]), _ptr(d), int(k), int(max_iters), _ptr(c))
        if it < 0:
            raise ValueError("oracle_kmeans_row: bad arguments")
        return c, int(it)

    def encode(self, w: np.ndarray, bits: int, fraction: float, max_iters: int,
               rows: Optional[np.ndarray] = None):
        """Encode fp16 weights [n_out, k_in]: returns dict with codes (canonical
        words of the requested rows), lut (fp16 bits of those rows), rowptr, col,
        val (S for all rows), iters (per requested row)."""
        w = _c(w, np.uint16)
        n_out, k_in = w.shape
        wpr = self.lib.oracle_words_per_row(k_in, bits)
        if wpr < 0:
            raise ValueError("K*bits must be a multiple of 32")
        rows_c = None if rows is None else _c(rows, np.int32)
        n_rows = n_out if rows_c is None else int(rows_c.shape[0])
        cap = 2 * self.outliers_per_tail(n_out * k_in, fraction)
        codes = np.zeros((n_rows, wpr), dtype=np.uint32)
        lut = np.zeros((n_rows, 1 << bits), dtype=np.uint16)
        rowptr = np.zeros(n_out + 1, dtype=np.int32)
        col = np.zeros(max(cap, 1), dtype=np.int32)
        val = np.zeros(max(cap, 1), dtype=np.uint16)
        nnz = ctypes.c_int64(0)
        iters = np.zeros(n_rows, dtype=np.int32)
        rc = self.lib.oracle_encode(n_out, k_in, bits, _ptr(w), float(fraction), int(max_iters), _ptr(rows_c), n_rows,
                                    _ptr(codes), _ptr(lut), _ptr(rowptr), _ptr(col), _ptr(val), max(cap, 1),
                                    ctypes.byref(nnz), _ptr(iters))
        if rc:
            raise ValueError("oracle_encode: bad arguments")
        n = int(nnz.value)
        return {"codes": codes, "lut": lut, "rowptr": rowptr, "col": col[:n].copy(), "val": val[:n].copy(),
                "iters": iters}

    def gemv_layer(self, layer, x, rows=None):
        return self.gemv(layer.n_out, layer.k_in, layer.bits, layer.codes, layer.lut, layer.rowptr,
                         layer.col, layer.val, x, rows)


def default() -> Oracle:
    return Oracle()
