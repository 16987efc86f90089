"""Python binding of ``libsqz.so`` (C ABI in ``include/sqz.h``).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Functions keep the C names.  Device arrays are torch CUDA tensors
(fp16 data may be passed as ``torch.float16`` or as its ``torch.int16`` bit
pattern); streams default to torch's current stream.  A non-OK status raises
:class:`SqzError` carrying the library's message.  If ``libsqz.so`` is
missing the first call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsqz.so")

SQZ_OK = 0
SQZ_ERR_INVALID_ARG = 1
SQZ_ERR_UNSUPPORTED = 2
SQZ_ERR_CUDA = 3
SQZ_ERR_OOM = 4
SQZ_ERR_TIMEOUT = 5
SQZ_MAX_BATCH = 16
SQZ_MAC_TENSOR_CORES = 0
SQZ_MAC_CUDA_CORES = 1
SQZ_MAC_MIXED = 2
SQZ_CSR_BALANCED = 0
SQZ_CSR_ROWWISE = 1

STATUS_NAMES = {0: "SQZ_OK", 1: "SQZ_ERR_INVALID_ARG", 2: "SQZ_ERR_UNSUPPORTED", 3: "SQZ_ERR_CUDA",
                4: "SQZ_ERR_OOM", 5: "SQZ_ERR_TIMEOUT"}

# Every entry point include/sqz.h declares.
EXPORTED = ("sqz_create_layer", "sqz_gemv", "sqz_gemv_host", "sqz_debug_dequant", "sqz_layer_info",
            "sqz_destroy", "sqz_fp16_gemv", "sqz_last_error", "sqz_version", "sqz_check_csr_static",
            "sqz_layer_set_mac", "sqz_layer_set_csr_mode", "sqz_layer_status", "sqz_encode",
            "sqz_encode_outliers", "sqz_plan_query", "sqz_layer_set_predecode", "sqz_tile_split_query")


class SqzError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class sqz_plan_info(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "fused", "columns_per_launch", "launches", "grid", "threads", "ctas_per_sm", "smem_bytes", "passes",
        "ring_stages", "csr_stage_entries", "predecode")]


class sqz_layer_desc(ctypes.Structure):
    _fields_ = [
        ("n_out", ctypes.c_int32),
        ("k_in", ctypes.c_int32),
        ("bits", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("lut", ctypes.c_void_p),
        ("nnz", ctypes.c_int64),
        ("rowptr", ctypes.c_void_p),
        ("col", ctypes.c_void_p),
        ("val", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsqz.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lut_dequant_gemv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.sqz_create_layer.argtypes = [ctypes.POINTER(sqz_layer_desc), P, ctypes.POINTER(P)]
        L.sqz_gemv.argtypes = [P, P, i32, i64, P, i64, P]
        L.sqz_gemv_host.argtypes = [P, P, i32, i64, P, i64, P]
        L.sqz_debug_dequant.argtypes = [P, P, P]
        L.sqz_layer_info.argtypes = [P, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                                     ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.sqz_destroy.argtypes = [P]
        L.sqz_fp16_gemv.argtypes = [P, i32, i32, i64, P, i32, i64, P, i64, P]
        for name in ("sqz_create_layer", "sqz_gemv", "sqz_gemv_host", "sqz_debug_dequant", "sqz_layer_info",
                     "sqz_destroy", "sqz_fp16_gemv"):
            getattr(L, name).restype = ctypes.c_int
        L.sqz_layer_set_mac.argtypes = [P, i32]
        L.sqz_layer_set_mac.restype = ctypes.c_int
        L.sqz_layer_set_csr_mode.argtypes = [P, i32]
        L.sqz_layer_set_csr_mode.restype = ctypes.c_int
        L.sqz_layer_set_predecode.argtypes = [P, i32]
        L.sqz_layer_set_predecode.restype = ctypes.c_int
        L.sqz_layer_status.argtypes = [P, P, ctypes.POINTER(i32)]
        L.sqz_layer_status.restype = ctypes.c_int
        L.sqz_check_csr_static.argtypes = [P, P, i32, i32, i64, P, ctypes.POINTER(i32)]
        L.sqz_check_csr_static.restype = ctypes.c_int
        L.sqz_encode.argtypes = [P, i32, i32, i32, ctypes.c_double, i32, P, P, P, P, P, i64,
                                 ctypes.POINTER(i64), P, P]
        L.sqz_encode.restype = ctypes.c_int
        L.sqz_plan_query.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(sqz_plan_info)]
        L.sqz_plan_query.restype = ctypes.c_int
        L.sqz_tile_split_query.argtypes = [P, i32, i32, i32, i32, P, ctypes.POINTER(i32)]
        L.sqz_tile_split_query.restype = ctypes.c_int
        L.sqz_encode_outliers.argtypes = [i64, ctypes.c_double]
        L.sqz_encode_outliers.restype = i64
        L.sqz_last_error.argtypes = []
        L.sqz_last_error.restype = ctypes.c_char_p
        L.sqz_version.argtypes = []
        L.sqz_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def sqz_last_error() -> str:
    return lib().sqz_last_error().decode("utf-8", "replace")


def sqz_version() -> int:
    return int(lib().sqz_version())


def _check(status: int, where: str) -> None:
    if status != SQZ_OK:
        raise SqzError(status, where, sqz_last_error())


def _dptr(t: Optional[torch.Tensor], name: str, dtypes) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() else None


def _hptr(t: torch.Tensor, name: str) -> Optional[int]:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype not in (torch.float16, torch.int16):
        raise TypeError(f"{name} must hold fp16 data")
    return t.data_ptr() if t.numel() else None


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


_H16 = (torch.float16, torch.int16)


def _lead(t: torch.Tensor, name: str) -> int:
    """Rows of a 2-D (or 1-D = one row) row-major tensor and its leading dimension."""
    if t.dim() == 1:
        return t.shape[0]
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 1-D or a 2-D row-major matrix")
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


class Layer:
    """Owning handle for an ``sqz_layer_t`` (destroyed on garbage collection)."""

    def __init__(self, handle: int, n_out: int, k_in: int, bits: int, nnz: int):
        self.handle = ctypes.c_void_p(handle)
        self.n_out, self.k_in, self.bits, self.nnz = n_out, k_in, bits, nnz

    def close(self) -> None:
        if self.handle is not None and self.handle.value:
            sqz_destroy(self)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def _as_parameter_(self):
        if self.handle is None:
            raise ValueError("layer has been destroyed")
        return self.handle


def sqz_create_layer(n_out: int, k_in: int, bits: int, codes: torch.Tensor, lut: torch.Tensor,
                     rowptr: Optional[torch.Tensor] = None, col: Optional[torch.Tensor] = None,
                     val: Optional[torch.Tensor] = None, stream=None) -> Layer:
    """Create a layer from canonical device arrays (see ``include/sqz.h``)."""
    nnz = 0 if col is None else int(col.numel())
    d = sqz_layer_desc(
        n_out=n_out, k_in=k_in, bits=bits,
        codes=_dptr(codes, "codes", (torch.int32, torch.uint32)),
        lut=_dptr(lut, "lut", _H16),
        nnz=nnz,
        rowptr=_dptr(rowptr, "rowptr", (torch.int32,)),
        col=_dptr(col, "col", (torch.int32,)),
        val=_dptr(val, "val", _H16),
    )
    out = ctypes.c_void_p()
    _check(lib().sqz_create_layer(ctypes.byref(d), _stream(stream), ctypes.byref(out)), "sqz_create_layer")
    return Layer(out.value, n_out, k_in, bits, nnz)


def _check_shapes(layer: Layer, x: torch.Tensor, y: torch.Tensor, batch: int) -> None:
    rows_x = x.shape[0] if x.dim() == 2 else 1
    rows_y = y.shape[0] if y.dim() == 2 else 1
    if x.shape[-1] < layer.k_in or y.shape[-1] < layer.n_out:
        raise ValueError(f"x needs >= {layer.k_in} columns and y >= {layer.n_out} (got {tuple(x.shape)}, "
                         f"{tuple(y.shape)})")
    if batch > rows_x or batch > rows_y:
        raise ValueError(f"batch {batch} exceeds the rows of x {tuple(x.shape)} or y {tuple(y.shape)}")


def sqz_gemv(layer: Layer, x: torch.Tensor, y: torch.Tensor, batch: Optional[int] = None, stream=None) -> None:
    """y[b, :N] = (Q + S) x[b, :K] for b < batch (device tensors, fp16)."""
    batch = (x.shape[0] if x.dim() == 2 else 1) if batch is None else batch
    _check_shapes(layer, x, y, batch)
    _check(lib().sqz_gemv(layer, _dptr_any(x, "x"), batch, _lead(x, "x"), _dptr_any(y, "y"), _lead(y, "y"),
                          _stream(stream)), "sqz_gemv")


def _dptr_any(t: torch.Tensor, name: str) -> Optional[int]:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in _H16:
        raise TypeError(f"{name} must hold fp16 data")
    return t.data_ptr() if t.numel() else None


def sqz_gemv_host(layer: Layer, x: torch.Tensor, y: torch.Tensor, batch: Optional[int] = None, stream=None) -> None:
    """Host-memory variant: x and y are CPU tensors (pinned for async copies)."""
    batch = (x.shape[0] if x.dim() == 2 else 1) if batch is None else batch
    _check_shapes(layer, x, y, batch)
    _check(lib().sqz_gemv_host(layer, _hptr(x, "x"), batch, _lead(x, "x"), _hptr(y, "y"), _lead(y, "y"),
                               _stream(stream)), "sqz_gemv_host")


def sqz_debug_dequant(layer: Layer, w_out: torch.Tensor, stream=None) -> None:
    _check(lib().sqz_debug_dequant(layer, _dptr(w_out, "w_out", _H16), _stream(stream)), "sqz_debug_dequant")


def sqz_layer_info(layer: Layer) -> dict:
    n, k, b = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    nnz, nbytes = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().sqz_layer_info(layer, ctypes.byref(n), ctypes.byref(k), ctypes.byref(b), ctypes.byref(nnz),
                                ctypes.byref(nbytes)), "sqz_layer_info")
    return dict(n_out=n.value, k_in=k.value, bits=b.value, nnz=nnz.value, device_bytes=nbytes.value)


def sqz_destroy(layer: Layer) -> None:
    h = layer.handle if isinstance(layer, Layer) else layer
    _check(lib().sqz_destroy(h), "sqz_destroy")
    if isinstance(layer, Layer):
        layer.handle = None


def sqz_fp16_gemv(w: torch.Tensor, x: torch.Tensor, y: torch.Tensor, batch: Optional[int] = None,
                  stream=None) -> None:
    """Dense fp16 yardstick: y = W x, W [N][ldw] fp16 on the device."""
    batch = (x.shape[0] if x.dim() == 2 else 1) if batch is None else batch
    n_out, k_in = w.shape
    _check(lib().sqz_fp16_gemv(_dptr_any(w, "w"), n_out, k_in, _lead(w, "w"), _dptr_any(x, "x"), batch,
                               _lead(x, "x"), _dptr_any(y, "y"), _lead(y, "y"), _stream(stream)), "sqz_fp16_gemv")


def create_layer_from_numpy(n_out: int, k_in: int, bits: int, codes, lut, rowptr=None, col=None, val=None,
                            device=None, stream=None) -> Layer:
    """Copy host (numpy) arrays in canonical storage to the device and create a layer."""
    import numpy as np

    dev = torch.device("cuda") if device is None else torch.device(device)

    def up(a, dt):
        if a is None:
            return None
        return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)

    nnz = 0 if col is None else len(col)
    t_codes = up(codes, np.int32)
    t_lut = up(lut, np.int16)
    t_rp = up(rowptr, np.int32) if nnz else None
    t_col = up(col, np.int32) if nnz else None
    t_val = up(val, np.int16) if nnz else None
    layer = sqz_create_layer(n_out, k_in, bits, t_codes, t_lut, t_rp, t_col, t_val, stream=stream)
    torch.cuda.current_stream(dev).synchronize()
    return layer


def sqz_check_csr_static(rowptr: Optional[torch.Tensor], col: Optional[torch.Tensor], n_out: int, k_in: int,
                         stream=None) -> int:
    """CSR check without device allocation; returns the flag word (0 = well formed)."""
    nnz = 0 if col is None else int(col.numel())
    flags = ctypes.c_int32(-1)
    _check(lib().sqz_check_csr_static(_dptr(rowptr, "rowptr", (torch.int32,)), _dptr(col, "col", (torch.int32,)),
                                      n_out, k_in, nnz, _stream(stream), ctypes.byref(flags)),
           "sqz_check_csr_static")
    return int(flags.value)


B200_DEVICE = {"sm_count": 148, "smem_per_sm": 233472, "smem_optin": 232448}


def sqz_plan_query(n_out: int, k_in: int, bits: int, batch: int, sm_count: int = 148, smem_per_sm: int = 233472,
                   smem_optin: int = 232448, predecode: int = 0) -> dict:
    """The launch plan sqz_gemv would use (host computation; defaults: B200)."""
    info = sqz_plan_info()
    _check(lib().sqz_plan_query(n_out, k_in, bits, batch, sm_count, smem_per_sm, smem_optin, int(predecode),
                                ctypes.byref(info)), "sqz_plan_query")
    return {name: int(getattr(info, name)) for name, _ in sqz_plan_info._fields_}


def sqz_tile_split_query(rowptr, n_out: int, k_in: int, bits: int, sm_count: int = 148):
    """The CTA -> tile split sqz_create_layer would use for this host rowptr
    (host computation): (first tile of every CTA plus the tile count as an
    int32 array of grid + 1 entries, True when the split by weight is used)."""
    rp = np.ascontiguousarray(rowptr, dtype=np.int32)
    if rp.shape != (n_out + 1,):
        raise ValueError(f"rowptr must have n_out + 1 = {n_out + 1} entries")
    ntiles = (max(n_out, 0) + 15) // 16
    first = np.zeros(max(1, min(sm_count, ntiles)) + 1, dtype=np.int32)
    weighted = ctypes.c_int32(0)
    _check(lib().sqz_tile_split_query(rp.ctypes.data, n_out, k_in, bits, sm_count, first.ctypes.data,
                                      ctypes.byref(weighted)), "sqz_tile_split_query")
    return first, bool(weighted.value)


def sqz_encode_outliers(n_weights: int, outlier_fraction: float) -> int:
    return int(lib().sqz_encode_outliers(int(n_weights), float(outlier_fraction)))


def sqz_encode(w: torch.Tensor, bits: int, outlier_fraction: float, max_iters: int, stream=None,
               want_iters: bool = False):
    """Quantize fp16 weights [n_out, k_in] (CUDA) into (codes, lut, rowptr, col,
    val[, iters]) device tensors in the layout sqz_create_layer takes."""
    if w.dim() != 2 or not w.is_contiguous():
        raise ValueError("w must be a contiguous [n_out, k_in] tensor")
    n_out, k_in = (int(d) for d in w.shape)
    dev = w.device
    nnz = sqz_encode_outliers(n_out * k_in, outlier_fraction)
    wpr = k_in * bits // 32 if bits in (3, 4) else 0
    codes = torch.empty((n_out, max(wpr, 1)), dtype=torch.int32, device=dev)
    lut = torch.empty((n_out, 1 << bits if bits in (3, 4) else 1), dtype=torch.int16, device=dev)
    rowptr = torch.empty(n_out + 1, dtype=torch.int32, device=dev)
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    val = torch.empty(max(nnz, 1), dtype=torch.int16, device=dev)
    iters = torch.empty(n_out, dtype=torch.int32, device=dev) if want_iters else None
    got = ctypes.c_int64(0)
    _check(lib().sqz_encode(_dptr_any(w, "w"), n_out, k_in, int(bits), float(outlier_fraction), int(max_iters),
                            codes.data_ptr(), lut.data_ptr(), rowptr.data_ptr(), col.data_ptr(), val.data_ptr(),
                            max(nnz, 1), ctypes.byref(got), None if iters is None else iters.data_ptr(),
                            _stream(stream)), "sqz_encode")
    n = int(got.value)
    out = (codes[:, :wpr], lut, rowptr, col[:n], val[:n])
    return out + (iters,) if want_iters else out


def sqz_layer_set_mac(layer: Layer, mac: int) -> None:
    _check(lib().sqz_layer_set_mac(layer, int(mac)), "sqz_layer_set_mac")


def sqz_layer_set_csr_mode(layer: Layer, mode: int) -> None:
    _check(lib().sqz_layer_set_csr_mode(layer, int(mode)), "sqz_layer_set_csr_mode")


def sqz_layer_set_predecode(layer: Layer, enable: int) -> None:
    _check(lib().sqz_layer_set_predecode(layer, int(enable)), "sqz_layer_set_predecode")


def sqz_layer_status(layer: Layer, stream=None) -> int:
    st = ctypes.c_int32(-1)
    _check(lib().sqz_layer_status(layer, _stream(stream), ctypes.byref(st)), "sqz_layer_status")
    return int(st.value)
