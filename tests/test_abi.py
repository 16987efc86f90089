"""The C ABI library loads, exports every entry point include/sqz.h declares,
and rejects bad arguments on the host with the documented status (no GPU
needed: these calls return before any CUDA call)."""
import ctypes
import os
import re

import pytest

from lut_dequant_gemv_b200 import binding as B
from lut_dequant_gemv_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sqz.h")).read()
    return sorted(set(re.findall(r"SQZ_API\s+[\w\s\*]+?\b(sqz_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_symbols() == sorted(B.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version(lib):
    assert B.sqz_version() >= 100


def _desc(**kw):
    d = dict(n_out=4, k_in=64, bits=3, codes=0x1000, lut=0x2000, nnz=0, rowptr=None, col=None, val=None)
    d.update(kw)
    return B.sqz_layer_desc(**d)


@pytest.mark.parametrize("kw,msg", [
    (dict(bits=2), "bits"),
    (dict(bits=5), "bits"),
    (dict(k_in=48, bits=3), "multiple of 32"),
    (dict(k_in=12, bits=4), "multiple of 8"),
    (dict(n_out=-1), "negative"),
    (dict(codes=None), "codes"),
    (dict(lut=None), "lut"),
    (dict(nnz=5, rowptr=0x3000, col=None, val=0x4000), "NULL"),
    (dict(nnz=-1), "nnz"),
    (dict(nnz=1 << 31), "nnz"),
])
def test_create_rejects_bad_descriptor(lib, kw, msg):
    out = ctypes.c_void_p(0x1234)
    st = lib.sqz_create_layer(ctypes.byref(_desc(**kw)), None, ctypes.byref(out))
    assert st == B.SQZ_ERR_INVALID_ARG
    assert out.value is None
    assert msg in B.sqz_last_error()


def test_create_rejects_null_desc(lib):
    out = ctypes.c_void_p()
    assert lib.sqz_create_layer(None, None, ctypes.byref(out)) == B.SQZ_ERR_INVALID_ARG
    assert lib.sqz_create_layer(ctypes.byref(_desc()), None, None) == B.SQZ_ERR_INVALID_ARG


def test_gemv_rejects_null_layer(lib):
    assert lib.sqz_gemv(None, 0x1000, 1, 64, 0x2000, 64, None) == B.SQZ_ERR_INVALID_ARG
    assert "layer" in B.sqz_last_error()
    assert lib.sqz_gemv_host(None, 0x1000, 1, 64, 0x2000, 64, None) == B.SQZ_ERR_INVALID_ARG
    assert lib.sqz_debug_dequant(None, 0x1000, None) == B.SQZ_ERR_INVALID_ARG
    assert lib.sqz_layer_info(None, None, None, None, None, None) == B.SQZ_ERR_INVALID_ARG


def test_destroy_accepts_null(lib):
    assert lib.sqz_destroy(None) == B.SQZ_OK


@pytest.mark.parametrize("args", [
    (0x1000, 4, 64, 64, 0x2000, 0, 64, 0x3000, 4),    # batch 0
    (0x1000, 4, 64, 64, 0x2000, 17, 64, 0x3000, 4),   # batch 17
    (0x1000, 4, 64, 32, 0x2000, 1, 64, 0x3000, 4),    # ldw < K
    (0x1000, 4, 64, 64, 0x2000, 1, 63, 0x3000, 4),    # ldx < K
    (0x1000, 4, 64, 64, 0x2000, 1, 64, 0x3000, 3),    # ldy < N
    (None, 4, 64, 64, 0x2000, 1, 64, 0x3000, 4),      # w NULL
    (0x1000, -4, 64, 64, 0x2000, 1, 64, 0x3000, 4),   # negative N
])
def test_fp16_gemv_rejects_bad_arguments(lib, args):
    assert lib.sqz_fp16_gemv(*args, None) == B.SQZ_ERR_INVALID_ARG


def test_layer_options_reject_null_handles_and_unknown_values(lib):
    assert lib.sqz_layer_set_mac(None, 0) == B.SQZ_ERR_INVALID_ARG
    assert lib.sqz_layer_set_csr_mode(None, B.SQZ_CSR_ROWWISE) == B.SQZ_ERR_INVALID_ARG
    assert "NULL" in B.sqz_last_error()


def test_encode_outlier_count_matches_the_oracle(lib, orc):
    # the count the caller sizes col/val with: 2 * floor(f * n / 2 + 1/2), at most n
    for n in (0, 1, 7, 1000, 4096 * 4096, 11008 * 4096):
        for f in (0.0, 0.004, 0.0045, 0.005, 0.5, 1.0):
            assert B.sqz_encode_outliers(n, f) == 2 * orc.outliers_per_tail(n, f), (n, f)
    assert B.sqz_encode_outliers(100, -0.1) == 0
    assert B.sqz_encode_outliers(100, float("nan")) == 0


@pytest.mark.parametrize("kw,msg", [
    (dict(w=None), "non-NULL"),
    (dict(bits=5), "bits"),
    (dict(n_out=0), "positive"),
    (dict(k_in=48), "multiple of 32"),
    (dict(fraction=1.5), "outlier_fraction"),
    (dict(fraction=float("nan")), "outlier_fraction"),
    (dict(iters=-1), "max_iters"),
    (dict(cap=3), "capacity"),
    (dict(col=None), "col and val"),
])
def test_encode_rejects_bad_arguments_before_touching_the_device(lib, kw, msg):
    import ctypes

    a = dict(w=0x1000, n_out=64, k_in=64, bits=3, fraction=0.01, iters=10, codes=0x2000, lut=0x3000,
             rowptr=0x4000, col=0x5000, val=0x6000, cap=1024)
    a.update(kw)
    nnz = ctypes.c_int64(-1)
    st = lib.sqz_encode(a["w"], a["n_out"], a["k_in"], a["bits"], a["fraction"], a["iters"], a["codes"], a["lut"],
                        a["rowptr"], a["col"], a["val"], a["cap"], ctypes.byref(nnz), None, None)
    assert st == B.SQZ_ERR_INVALID_ARG
    assert msg in B.sqz_last_error()
    assert nnz.value == 0
