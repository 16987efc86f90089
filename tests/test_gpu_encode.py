"""The encoder (sqz_encode) against the oracle's encoder, bit for bit.

Outlier set, CSR arrays, fp16 LUTs, packed codes and the iterations each
row ran are integer or bit-pattern results decided by exact comparisons
(order keys, fp64 distances of fp16 values, exact integer sums), so they
must be identical -- not close.  The layers are synthetic Student-t weights
("SqueezeLLM" summary page: weights are concentrated with a few extreme
values); ties at the thresholds, negative zeros, an all-zero matrix and a
zero fraction exercise the exact tie rules.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from lut_dequant_gemv_b200 import binding, build

    build.build()
    binding.lib()
    return binding


def gpu_encode(B, w_bits, bits, frac, iters):
    w = torch.from_numpy(w_bits.view(np.int16).copy()).cuda()
    codes, lut, rowptr, col, val, it = B.sqz_encode(w, bits, frac, iters, want_iters=True)
    torch.cuda.synchronize()
    host = lambda t: t.cpu().numpy()
    return {"codes": host(codes).view(np.uint32), "lut": host(lut).view(np.uint16), "rowptr": host(rowptr),
            "col": host(col), "val": host(val).view(np.uint16), "iters": host(it)}


def assert_same(g, o, rows=None, what=""):
    for k in ("rowptr", "col", "val"):
        assert np.array_equal(g[k], o[k]), (what, k)
    sel = slice(None) if rows is None else rows
    for k in ("codes", "lut", "iters"):
        gk = g[k][sel]
        assert np.array_equal(gk, o[k]), (what, k, int((gk != o[k]).sum()))


CASES = [
    # (name, n_out, k_in, bits, fraction, iters)
    ("3bit-small", 37, 256, 3, 0.0045, 40),
    ("4bit-ragged", 29, 200, 4, 0.01, 40),
    ("3bit-wide", 8, 4096, 3, 0.004, 60),
    ("4bit-noout", 16, 512, 4, 0.0, 30),
    ("3bit-noiter", 16, 256, 3, 0.02, 0),
    ("4bit-oneiter", 16, 256, 4, 0.02, 1),
]


@pytest.mark.parametrize("name,n_out,k_in,bits,frac,iters", CASES, ids=[c[0] for c in CASES])
def test_encode_matches_oracle(B, orc, name, n_out, k_in, bits, frac, iters):
    w = synth.make_weights(n_out, k_in, seed=3, key=name)
    g = gpu_encode(B, w, bits, frac, iters)
    o = orc.encode(w.reshape(n_out, k_in), bits, frac, iters)
    assert_same(g, o, what=name)
    assert g["rowptr"][-1] == B.sqz_encode_outliers(n_out * k_in, frac)


def test_encode_threshold_ties_and_signed_zeros(B, orc):
    """Weights from a small set of values: long runs of equal values at both
    thresholds (ranks in position order decide), and -0 mixed with +0."""
    rng = np.random.default_rng(9)
    pool = (np.arange(-24, 25) / 512.0).astype(np.float16)
    w = rng.choice(pool, size=(40, 320)).astype(np.float16)
    w[rng.random(w.shape) < 0.05] = np.float16(-0.0)
    for bits, frac in ((3, 0.05), (4, 0.2), (3, 1.0)):
        g = gpu_encode(B, w.view(np.uint16), bits, frac, 50)
        o = orc.encode(w.view(np.uint16), bits, frac, 50)
        assert_same(g, o, what=f"ties b{bits} f{frac}")


def test_encode_all_equal_weights(B, orc):
    for val in (0.0, -0.0, 0.125):
        w = np.full((8, 64), val, dtype=np.float16).view(np.uint16)
        g = gpu_encode(B, w, 3, 0.1, 10)
        o = orc.encode(w, 3, 0.1, 10)
        assert_same(g, o, what=f"constant {val}")


def test_encode_full_layer_sampled_rows(B, orc):
    """A 4096x4096 layer at 0.45 % outliers: the whole outlier set and CSR
    against the oracle, and the k-means of 48 rows (first, last, random)."""
    n_out, k_in = 4096, 4096
    w = synth.make_weights(n_out, k_in, seed=5, key="enc-full")
    g = gpu_encode(B, w, 3, 0.0045, 40)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, n_out - 1], rng.choice(n_out, 45, replace=False)])).astype(np.int32)
    o = orc.encode(w.reshape(n_out, k_in), 3, 0.0045, 40, rows=rows)
    assert_same(g, o, rows=rows, what="full")


def test_encoded_layer_runs_through_the_gemv(B, orc):
    """Encode, create the layer from the encoder's device outputs, and run the
    fused GEMV: parity with the oracle GEMV of the oracle's encoding, and the
    product close to the unquantized W x (quantization error only)."""
    n_out, k_in, bits = 512, 1024, 4
    w = synth.make_weights(n_out, k_in, seed=6, key="enc-gemv")
    wt = torch.from_numpy(w.view(np.int16).copy()).cuda()
    codes, lut, rowptr, col, val = B.sqz_encode(wt, bits, 0.0045, 40)
    layer = B.sqz_create_layer(n_out, k_in, bits, codes, lut, rowptr, col, val)
    x = synth.make_x(2, k_in, seed=6, key="enc-gemv")
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    y = torch.empty((2, n_out), dtype=torch.int16, device="cuda")
    B.sqz_gemv(layer, xd, y)
    torch.cuda.synchronize()
    yg = y.cpu().numpy().view(np.float16).astype(np.float64)
    o = orc.encode(w.reshape(n_out, k_in), bits, 0.0045, 40)
    y_ref, bound = orc.gemv(n_out, k_in, bits, o["codes"], o["lut"], o["rowptr"], o["col"], o["val"], x)
    assert np.all(np.abs(yg - y_ref) <= 1e-3 * bound + 1e-6)
    wd = w.view(np.float16).astype(np.float64).reshape(n_out, k_in)
    xf = x.view(np.float16).astype(np.float64)
    dense = xf @ wd.T
    rel = np.linalg.norm(yg - dense) / np.linalg.norm(dense)
    assert rel < 0.2, rel


def test_encode_rejects_bad_inputs(B):
    w = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    w[1, 3] = float("nan")
    with pytest.raises(B.SqzError) as e:
        B.sqz_encode(w, 3, 0.01, 5)
    assert e.value.status == B.SQZ_ERR_INVALID_ARG
    big = torch.full((2, 16384), 65504.0, dtype=torch.float16, device="cuda")  # 16384 * 65504 > 2^29
    with pytest.raises(B.SqzError) as e:
        B.sqz_encode(big, 4, 0.0, 5)
    assert e.value.status == B.SQZ_ERR_UNSUPPORTED
