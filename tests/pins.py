"""Pins for the CPU oracle: checks against facts that do not come from the
oracle itself -- exact rational brute force, library routines (numpy matmul,
scipy CSR products, numpy's fp16 conversion), closed forms, invariants and
the values the pages print.

Each ``pin_*`` function takes an oracle instance and raises AssertionError
on a mismatch; ``tests/test_oracle_pins.py`` runs them against the real
oracle and ``tests/test_oracle_mutants.py`` runs them against deliberately
broken copies to show that each plausible mistake is caught.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers ---

def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def f16_bits(vals) -> np.ndarray:
    return np.asarray(vals, dtype=np.float64).astype(np.float16).view(np.uint16)


def f16_val(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bigint_codes(words_row: np.ndarray, bits: int, k_in: int):
    """Independent reader: treat the row as one little-endian big integer."""
    big = 0
    for i, w in enumerate(words_row.tolist()):
        big |= int(w) << (32 * i)
    mask = (1 << bits) - 1
    return [(big >> (k * bits)) & mask for k in range(k_in)]


def bigint_pack(codes_row, bits: int) -> np.ndarray:
    big = 0
    for k, c in enumerate(codes_row):
        big |= int(c) << (k * bits)
    nwords = len(codes_row) * bits // 32
    return np.array([(big >> (32 * i)) & 0xFFFFFFFF for i in range(nwords)], dtype=np.uint32)


def exact_dense_plus_sparse(codes, lut, rowptr, col, val, x, n_out, k_in, bits):
    """Brute force with exact rationals: densify W = lut[code] + S (duplicate
    CSR entries summed), then y = W x."""
    L = 1 << bits
    W = [[Fraction(0)] * k_in for _ in range(n_out)]
    for i in range(n_out):
        cs = bigint_codes(codes[i], bits, k_in)
        for k in range(k_in):
            W[i][k] += Fraction(float(f16_val(lut[i * L + cs[k]] if lut.ndim == 1 else lut[i, cs[k]])))
    if col is not None and len(col):
        for i in range(n_out):
            for j in range(int(rowptr[i]), int(rowptr[i + 1])):
                W[i][int(col[j])] += Fraction(float(f16_val(val[j])))
    xs = [[Fraction(float(v)) for v in f16_val(xb)] for xb in x]
    y = [[sum((W[i][k] * xb[k] for k in range(k_in)), Fraction(0)) for i in range(n_out)] for xb in xs]
    return y


def random_csr(rng, n_out, k_in, nnz, dup=False, unsorted=False, dyadic=False):
    rows = np.sort(rng.integers(0, n_out, size=nnz))
    col = rng.integers(0, k_in, size=nnz).astype(np.int32)
    if not dup:
        # re-draw until (row, col) pairs are unique
        seen = set()
        for j in range(nnz):
            while (int(rows[j]), int(col[j])) in seen:
                col[j] = rng.integers(0, k_in)
            seen.add((int(rows[j]), int(col[j])))
    rowptr = np.zeros(n_out + 1, dtype=np.int32)
    np.cumsum(np.bincount(rows, minlength=n_out), out=rowptr[1:])
    if not unsorted:
        for i in range(n_out):
            a, b = rowptr[i], rowptr[i + 1]
            col[a:b] = np.sort(col[a:b])
    if dyadic:
        val = f16_bits(rng.integers(-64, 65, size=nnz) / 256.0)
    else:
        val = f16_bits(rng.choice([-1, 1], size=nnz) * rng.uniform(0.1, 0.5, size=nnz))
    return rowptr, col, val


def tiny_case(seed, n_out, k_in, bits, batch, nnz, dyadic=True, dup=False, unsorted=False):
    rng = np.random.default_rng(seed)
    L = 1 << bits
    code_mat = rng.integers(0, L, size=(n_out, k_in))
    codes = np.stack([bigint_pack(code_mat[i], bits) for i in range(n_out)])
    if dyadic:
        lut = f16_bits(rng.integers(-40, 41, size=(n_out, L)) / 256.0)
        x = f16_bits(rng.integers(-8, 9, size=(batch, k_in)) / 8.0)
    else:
        lut = f16_bits(np.sort(rng.normal(0, 0.02, size=(n_out, L)), axis=1))
        x = f16_bits(rng.standard_normal(size=(batch, k_in)))
    rowptr, col, val = random_csr(rng, n_out, k_in, nnz, dup=dup, unsorted=unsorted, dyadic=dyadic)
    return code_mat, codes, lut, rowptr, col, val, x


# ------------------------------------------------------------------- pins ---

def pin_half_decode_all_patterns(orc):
    """The oracle's binary16 decoder equals numpy's conversion on all 2^16 patterns."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(h)) for h in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_unpack_bigint(orc):
    """P-6: unpack equals an independent big-integer bit reader."""
    rng = np.random.default_rng(11)
    for bits in (3, 4):
        for k_in in (32, 64, 96, 160, 1024):
            n_out = 3
            wpr = k_in * bits // 32
            words = rng.integers(0, 1 << 32, size=(n_out, wpr), dtype=np.uint64).astype(np.uint32)
            got = orc.unpack(words, n_out, k_in, bits)
            for i in range(n_out):
                assert got[i].tolist() == bigint_codes(words[i], bits, k_in), (bits, k_in, i)


def pin_pack_roundtrip(orc):
    """P-5: pack(unpack(w)) == w and unpack(pack(c)) == c, and pack matches
    the independent big-integer packer."""
    rng = np.random.default_rng(12)
    for bits in (3, 4):
        k_in = 256
        words = rng.integers(0, 1 << 32, size=(4, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
        cm = orc.unpack(words, 4, k_in, bits)
        assert np.array_equal(orc.pack(cm, bits), words)
        cm2 = rng.integers(0, 1 << bits, size=(4, k_in)).astype(np.uint8)
        packed = orc.pack(cm2, bits)
        assert np.array_equal(orc.unpack(packed, 4, k_in, bits), cm2)
        for i in range(4):
            assert np.array_equal(packed[i], bigint_pack(cm2[i].tolist(), bits))


def pin_straddling_codes(orc):
    """3-bit codes 10 and 21 of each 32-code group straddle word boundaries:
    code 10 occupies stream bits 30..32, code 21 bits 63..65."""
    cm = np.zeros((1, 32), dtype=np.uint8)
    cm[0, 10] = 0b101
    cm[0, 21] = 0b110
    w = orc.pack(cm, 3)[0]
    assert (w[0] >> 30) & 1 == 1 and (w[0] >> 31) & 1 == 0 and w[1] & 1 == 1
    assert (w[1] >> 31) & 1 == 0 and w[2] & 1 == 1 and (w[2] >> 1) & 1 == 1
    assert int(w[0]) == (1 << 30) and int(w[1]) == 1 and int(w[2]) == 0b11
    assert orc.unpack(w[None, :], 1, 32, 3)[0].tolist() == cm[0].tolist()


def pin_pack_density(orc):
    """The pages: 8 three-bit indices occupy 3 bytes (no padding)."""
    for bits, n_idx, n_bytes in ((int(a), int(b), int(c)) for a, b, c in read_golden("pack_density.txt")):
        k_in = 32 * n_idx  # whole words
        assert orc.lib.oracle_words_per_row(k_in, bits) * 4 == n_bytes * k_in // n_idx


def pin_bruteforce_exact(orc):
    """P-1: on tiny dyadic inputs every fp64 sum is exact, so the oracle must
    equal the exact rational brute force bit for bit (duplicates, unsorted
    columns, empty rows, padded x rows included)."""
    cases = [
        dict(seed=1, n_out=4, k_in=32, bits=3, batch=1, nnz=5),
        dict(seed=2, n_out=5, k_in=64, bits=4, batch=3, nnz=9, dup=True, unsorted=True),
        dict(seed=3, n_out=8, k_in=64, bits=3, batch=2, nnz=0),
        dict(seed=4, n_out=7, k_in=32, bits=4, batch=2, nnz=12, dup=True),
        dict(seed=5, n_out=3, k_in=96, bits=3, batch=3, nnz=7, unsorted=True),
    ]
    for c in cases:
        code_mat, codes, lut, rowptr, col, val, x = tiny_case(**c)
        exact = exact_dense_plus_sparse(codes, lut, rowptr, col, val, x, c["n_out"], c["k_in"], c["bits"])
        # x passed with a leading dimension larger than K
        ldx = c["k_in"] + 5
        xp = np.zeros((c["batch"], ldx), dtype=np.uint16)
        xp[:, :c["k_in"]] = x
        xp[:, c["k_in"]:] = f16_bits(1000.0)
        y, _ = orc.gemv(c["n_out"], c["k_in"], c["bits"], codes, lut, rowptr, col, val, xp)
        for b in range(c["batch"]):
            for i in range(c["n_out"]):
                assert Fraction(float(y[b, i])) == exact[b][i], (c, b, i)


def pin_bruteforce_fp16(orc):
    """P-1: random fp16 inputs agree with exact arithmetic to 1e-12 relative."""
    for seed, bits in ((21, 3), (22, 4)):
        n_out, k_in, batch = 6, 64, 2
        code_mat, codes, lut, rowptr, col, val, x = tiny_case(seed, n_out, k_in, bits, batch, 10, dyadic=False)
        exact = exact_dense_plus_sparse(codes, lut, rowptr, col, val, x, n_out, k_in, bits)
        y, bound = orc.gemv(n_out, k_in, bits, codes, lut, rowptr, col, val, x)
        for b in range(batch):
            for i in range(n_out):
                assert abs(Fraction(float(y[b, i])) - exact[b][i]) <= Fraction(1e-12) * Fraction(float(bound[b, i]))


def pin_bound_definition(orc):
    """bound(i,b) = sum of |terms|; with all-positive inputs it equals y."""
    rng = np.random.default_rng(31)
    n_out, k_in, bits = 4, 64, 4
    cm = rng.integers(0, 16, size=(n_out, k_in)).astype(np.uint8)
    codes = orc.pack(cm, bits)
    lut = f16_bits(rng.integers(1, 40, size=(n_out, 16)) / 256.0)
    x = f16_bits(rng.integers(1, 9, size=(1, k_in)) / 8.0)
    rowptr, col, val = random_csr(rng, n_out, k_in, 6, dyadic=True)
    val = f16_bits(np.abs(f16_val(val)) + 1.0 / 256)
    y, bound = orc.gemv(n_out, k_in, bits, codes, lut, rowptr, col, val, x)
    assert np.array_equal(y, bound)
    # sign flip of x: y negates, bound unchanged
    xn = f16_bits(-f16_val(x))
    y2, bound2 = orc.gemv(n_out, k_in, bits, codes, lut, rowptr, col, val, xn)
    assert np.array_equal(y2, -y) and np.array_equal(bound2, bound)


def pin_nnz0_equals_dense(orc):
    """P-2: with nnz = 0 the result is the textbook dense product W x,
    W = lut[code] (numpy matmul on independently unpacked codes)."""
    rng = np.random.default_rng(41)
    for bits in (3, 4):
        n_out, k_in, batch = 16, 256, 3
        words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
        lut = f16_bits(np.sort(rng.normal(0, 0.02, size=(n_out, 1 << bits)), axis=1))
        x = f16_bits(rng.standard_normal(size=(batch, k_in)))
        W = np.array([[f16_val(lut[i, c]) for c in bigint_codes(words[i], bits, k_in)] for i in range(n_out)])
        ref = f16_val(x) @ W.T
        y, bound = orc.gemv(n_out, k_in, bits, words, lut, None, None, None, x)
        assert np.all(np.abs(y - ref) <= 1e-12 * bound)


def pin_zero_lut_equals_scipy_csr(orc):
    """P-2: with an all-zero LUT the result is the textbook CSR product S x
    (scipy.sparse, which also sums duplicates and accepts unsorted columns)."""
    import scipy.sparse as sp

    rng = np.random.default_rng(42)
    n_out, k_in, batch, bits = 12, 128, 2, 3
    words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
    lut = np.zeros((n_out, 8), dtype=np.uint16)
    rowptr, col, val = random_csr(rng, n_out, k_in, 40, dup=True, unsorted=True)
    x = f16_bits(rng.standard_normal(size=(batch, k_in)))
    S = sp.csr_matrix((f16_val(val), col, rowptr), shape=(n_out, k_in))
    ref = (S @ f16_val(x).T).T
    y, bound = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
    assert np.all(np.abs(y - ref) <= 1e-12 * bound + 1e-300)


def pin_uniform_lut_closed_form(orc):
    """P-3: a LUT of uniformly spaced centroids a + j d reproduces uniform
    dequantization: y_i = a sum(x) + d sum_k code(i,k) x_k (+ S x)."""
    rng = np.random.default_rng(51)
    for bits in (3, 4):
        n_out, k_in = 6, 128
        d = 2.0 ** -7
        a = -(2 ** (bits - 1)) * d
        lut = np.tile(f16_bits(a + d * np.arange(1 << bits)), (n_out, 1))
        cm = rng.integers(0, 1 << bits, size=(n_out, k_in))
        words = np.stack([bigint_pack(cm[i].tolist(), bits) for i in range(n_out)])
        xm = rng.integers(-8, 9, size=k_in)
        x = f16_bits(xm / 8.0)[None, :]
        rowptr, col, val = random_csr(rng, n_out, k_in, 9, dyadic=True)
        y, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
        for i in range(n_out):
            exp = Fraction(a) * Fraction(int(xm.sum()), 8) + Fraction(d) * Fraction(int(cm[i] @ xm), 8)
            for j in range(rowptr[i], rowptr[i + 1]):
                exp += Fraction(float(f16_val(val[j]))) * Fraction(int(xm[col[j]]), 8)
            assert Fraction(float(y[0, i])) == exp


def pin_page_uniform_grid(orc):
    """P-3 on the pages' worked example: 8 uniform bins over [-0.5, 0.5]
    (printed centres and width 0.143).  The grid formula reproduces the
    printed values; with that grid (rounded to fp16) as every row's LUT the
    oracle equals uniform dequantization within the fp16 rounding of the grid."""
    g = {r[0]: r[1:] for r in read_golden("uniform_grid_3bit.txt")}
    w_min, w_max, k = float(g["w_min"][0]), float(g["w_max"][0]), int(g["k"][0])
    printed = [float(v) for v in g["values"]]
    q = [Fraction(w_min) + (j - 1) * (Fraction(w_max) - Fraction(w_min)) / (k - 1) for j in range(1, k + 1)]
    for qj, pj in zip(q, printed):
        assert abs(float(qj) - pj) <= 0.0005
    assert abs(float(q[1] - q[0]) - float(g["width"][0])) <= 0.0005
    rng = np.random.default_rng(52)
    n_out, k_in = 4, 64
    lut_row = f16_bits([float(v) for v in q])
    lut = np.tile(lut_row, (n_out, 1))
    cm = rng.integers(0, 8, size=(n_out, k_in))
    words = np.stack([bigint_pack(cm[i].tolist(), 3) for i in range(n_out)])
    x = f16_bits(rng.standard_normal(size=(1, k_in)))
    xv = [Fraction(float(v)) for v in f16_val(x[0])]
    y, _ = orc.gemv(n_out, k_in, 3, words, lut, None, None, None, x)
    rounding = max(abs(Fraction(float(f16_val(lut_row[j]))) - q[j]) for j in range(8))
    for i in range(n_out):
        exp = sum((q[int(cm[i, kk])] * xv[kk] for kk in range(k_in)), Fraction(0))
        tol = rounding * sum(abs(v) for v in xv) + Fraction(1, 10 ** 12)
        assert abs(Fraction(float(y[0, i])) - exp) <= tol


def pin_constant_code_rows(orc):
    """P-4: all codes of row i equal c_i  =>  y_i = lut[i][c_i] * sum_k x_k (+ S row)."""
    rng = np.random.default_rng(61)
    for bits in (3, 4):
        n_out, k_in = 8, 96 if bits == 3 else 64
        c = rng.integers(0, 1 << bits, size=n_out)
        cm = np.repeat(c[:, None], k_in, axis=1)
        words = np.stack([bigint_pack(cm[i].tolist(), bits) for i in range(n_out)])
        lut = f16_bits(rng.integers(-40, 41, size=(n_out, 1 << bits)) / 256.0)
        xm = rng.integers(-8, 9, size=(2, k_in))
        x = f16_bits(xm / 8.0)
        rowptr, col, val = random_csr(rng, n_out, k_in, 11, dyadic=True)
        y, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
        for b in range(2):
            for i in range(n_out):
                exp = Fraction(float(f16_val(lut[i, c[i]]))) * Fraction(int(xm[b].sum()), 8)
                for j in range(rowptr[i], rowptr[i + 1]):
                    exp += Fraction(float(f16_val(val[j]))) * Fraction(int(xm[b, col[j]]), 8)
                assert Fraction(float(y[b, i])) == exp


def pin_power_of_two_scaling(orc):
    """P-5: y(2^e x) = 2^e y(x) exactly (fp64 scaling by powers of two is exact)."""
    rng = np.random.default_rng(71)
    n_out, k_in, bits = 10, 128, 3
    words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
    lut = f16_bits(np.sort(rng.normal(0, 0.02, size=(n_out, 8)), axis=1))
    rowptr, col, val = random_csr(rng, n_out, k_in, 15)
    xv = rng.choice([-1, 1], size=(1, k_in)) * rng.uniform(2.0 ** -5, 2.0 ** 3, size=(1, k_in))
    x = f16_bits(xv)
    y, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
    for e in (-3, 4):
        xs = f16_bits(f16_val(x) * 2.0 ** e)
        assert np.array_equal(f16_val(xs), f16_val(x) * 2.0 ** e)
        ys, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, xs)
        assert np.array_equal(ys, y * 2.0 ** e)


def pin_batch_columns(orc):
    """P-5: batch column b equals the batch-1 result for x_b."""
    rng = np.random.default_rng(81)
    n_out, k_in, bits, batch = 9, 64, 4, 4
    words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
    lut = f16_bits(np.sort(rng.normal(0, 0.02, size=(n_out, 16)), axis=1))
    rowptr, col, val = random_csr(rng, n_out, k_in, 12)
    x = f16_bits(rng.standard_normal(size=(batch, k_in)))
    y, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
    for b in range(batch):
        yb, _ = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x[b:b + 1])
        assert np.array_equal(yb[0], y[b])


def pin_row_subset(orc):
    """Evaluating a subset of rows gives the same values as the full evaluation."""
    rng = np.random.default_rng(82)
    n_out, k_in, bits = 20, 64, 3
    words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
    lut = f16_bits(np.sort(rng.normal(0, 0.02, size=(n_out, 8)), axis=1))
    rowptr, col, val = random_csr(rng, n_out, k_in, 30)
    x = f16_bits(rng.standard_normal(size=(2, k_in)))
    y, b = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x)
    rows = np.array([19, 0, 7, 7, 3], dtype=np.int32)
    ys, bs = orc.gemv(n_out, k_in, bits, words, lut, rowptr, col, val, x, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(bs, b[:, rows])


def pin_dequant_lookup(orc):
    """w(i,k) = lut[i][code(i,k)] bit for bit (independent reader + numpy indexing)."""
    rng = np.random.default_rng(91)
    for bits in (3, 4):
        n_out, k_in = 5, 160
        words = rng.integers(0, 1 << 32, size=(n_out, k_in * bits // 32), dtype=np.uint64).astype(np.uint32)
        lut = rng.integers(0, 1 << 16, size=(n_out, 1 << bits), dtype=np.uint32).astype(np.uint16)
        w = orc.dequant(words, lut, n_out, k_in, bits)
        for i in range(n_out):
            assert w[i].tolist() == [int(lut[i, c]) for c in bigint_codes(words[i], bits, k_in)]


def pin_csr_checks(orc):
    """Malformed CSR (rowptr[0] != 0, decreasing rowptr, rowptr[N] != nnz,
    column outside [0, K)) is rejected; empty rows and nnz = 0 are accepted."""
    rp = np.array([0, 2, 2, 3], dtype=np.int32)
    col = np.array([1, 5, 0], dtype=np.int32)
    assert orc.check_csr(3, 8, rp, col)
    assert orc.check_csr(3, 8, None, None)
    assert not orc.check_csr(3, 8, np.array([1, 2, 2, 3], dtype=np.int32), col)
    assert not orc.check_csr(3, 8, np.array([0, 2, 1, 3], dtype=np.int32), col)
    assert not orc.check_csr(3, 8, np.array([0, 2, 2, 2], dtype=np.int32), col)
    assert not orc.check_csr(3, 8, rp, np.array([1, 8, 0], dtype=np.int32))
    assert not orc.check_csr(3, 8, rp, np.array([1, -1, 0], dtype=np.int32))


# ------------------------------------------------------------ encoder pins ---
# The encoder ("SqueezeLLM" summary page: Eq. 1 k-means and the
# Dense-and-Sparse decomposition) checked against numpy's fp16 rounding,
# numpy's sort, scikit-learn's Lloyd k-means, exact rational arithmetic and
# the uniform grid the page prints.

def pin_enc_double_to_half_matches_numpy(orc):
    rng = np.random.default_rng(41)
    vals = rng.standard_normal(20000) * np.exp(rng.uniform(-22, 12, 20000))
    edge = [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -24, 2.0 ** -14,
            2.0 ** -14 - 2.0 ** -25, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1 / 3, -2.5e-8]
    vals = np.concatenate([vals, edge, -np.array(edge)])
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([orc.double_to_half(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want), int((got != want).sum())


def pin_enc_outlier_tails_page_example(orc):
    # the page's 0.2th / 99.8th percentiles: 0.4 % of the weights, 0.2 % in each tail
    lo, hi, frac, tail = (float(v) for v in read_golden("outlier_percentiles.txt")[0])
    assert abs((lo + (100.0 - hi)) / 100.0 - frac) < 1e-12 and abs(lo / 100.0 - tail) < 1e-12
    n = 100000
    assert orc.outliers_per_tail(n, frac) == round(tail * n) == 200
    assert orc.outliers_per_tail(1000, 0.0045) == 2  # 2.25 rounds to 2
    assert orc.outliers_per_tail(1000, 0.005) == 3   # 2.5 rounds up (the reading taken)
    assert orc.outliers_per_tail(10, 1.0) == 5        # at most half the weights per tail


def pin_enc_outlier_selection_is_order_statistics(orc):
    rng = np.random.default_rng(42)
    # values from a small set so that the thresholds fall inside runs of ties
    pool = (np.arange(-40, 41) / 64.0).astype(np.float16)
    w = rng.choice(pool, size=(24, 96), p=None).astype(np.float16)
    w[rng.integers(0, 24, 6), rng.integers(0, 96, 6)] = np.float16(-0.0)
    n = w.size
    for m in (0, 1, 7, 37, 200):
        marks = orc.select_outliers(w.view(np.uint16), m).ravel()
        v = w.astype(np.float64).ravel() + 0.0
        order = np.lexsort((np.arange(n), v))  # numpy sort by value, then position
        want = np.zeros(n, dtype=np.uint8)
        want[order[:m]] = 1
        want[order[n - m:]] = 1
        assert np.array_equal(marks, want), m
        assert int(marks.sum()) == 2 * m
        if m:
            lo_sel, hi_sel = order[:m], order[n - m:]
            rest = v[marks == 0]
            assert v[lo_sel].max() <= rest.min() and rest.max() <= v[hi_sel].min()


def pin_enc_kmeans_page_uniform_init(orc):
    g = {r[0]: r[1:] for r in read_golden("uniform_grid_3bit.txt")}
    lo, hi, k = float(g["w_min"][0]), float(g["w_max"][0]), int(g["k"][0])
    d = np.linspace(lo, hi, 101)
    c, it = orc.kmeans_row(d, k, 0)
    assert it == 0
    assert np.allclose(c, [float(t) for t in g["values"]], atol=5e-4)
    assert abs((c[1] - c[0]) - float(g["width"][0])) < 5e-4


def pin_enc_kmeans_empty_clusters_keep_place(orc):
    # clusters 1..6 of the grid over [0, 1] get no values: they stay where
    # they started, the two others settle on the means 0 and 1
    d = np.array([0.0, 0.0, 0.0, 1.0])
    c, it = orc.kmeans_row(d, 8, 10)
    assert it <= 2
    assert np.allclose(c, np.array([j / 7.0 for j in range(8)]), rtol=0, atol=1e-15)
    assert c[0] == 0.0 and c[7] == 1.0


def pin_enc_kmeans_matches_sklearn(orc):
    from sklearn.cluster import KMeans

    rng = np.random.default_rng(43)
    for k in (8, 16):
        # one tight group of values near each point of the starting grid (no
        # cluster ever empties, where the two implementations would differ)
        grid = np.linspace(-0.05, 0.05, k)
        centres = grid + rng.uniform(-0.2, 0.2, k) * (grid[1] - grid[0])
        centres[0], centres[-1] = grid[0], grid[-1]
        d = np.concatenate([c0 + rng.standard_normal(64) * 2e-4 for c0 in centres])
        d = d.astype(np.float16).astype(np.float64)
        c, it = orc.kmeans_row(d, k, 100)
        init = d.min() + np.arange(k) * ((d.max() - d.min()) / (k - 1))
        km = KMeans(n_clusters=k, init=init.reshape(-1, 1), n_init=1, max_iter=100, tol=0.0,
                    algorithm="lloyd").fit(d.reshape(-1, 1))
        ref = np.sort(km.cluster_centers_.ravel())
        assert it < 100
        assert np.allclose(np.sort(c), ref, rtol=0, atol=1e-12), (k, np.abs(np.sort(c) - ref).max())


def pin_enc_kmeans_fixed_point_exact(orc):
    rng = np.random.default_rng(44)
    d = (rng.standard_normal(300) * 0.02).astype(np.float16).astype(np.float64)
    c, it = orc.kmeans_row(d, 8, 200)
    assert it < 200
    cf = [Fraction(x) for x in c]
    groups = [[] for _ in range(8)]
    for v in d:
        fv = Fraction(v)
        dist = [abs(fv - cj) for cj in cf]
        groups[dist.index(min(dist))].append(fv)
    for j in range(8):
        if groups[j]:
            mean = sum(groups[j]) / len(groups[j])
            assert abs(float(mean) - c[j]) <= 2.0 ** -52 * abs(c[j]), j


def pin_enc_kmeans_sse_nonincreasing(orc):
    rng = np.random.default_rng(45)
    d = (rng.standard_t(4, 512) * 0.02).astype(np.float16).astype(np.float64)
    prev = None
    for t in range(0, 8):
        c, _ = orc.kmeans_row(d, 8, t)
        sse = float(np.min((d[:, None] - c[None, :]) ** 2, axis=1).sum())
        if prev is not None:
            assert sse <= prev * (1 + 1e-12), t
        prev = sse


def pin_enc_codes_are_nearest_fp16_entry(orc):
    # a wider layer: every code must index the nearest entry of the row's
    # fp16 LUT (fp16 - fp16 differences are exact in fp64; argmin takes the
    # lowest index on a tie), which the codes of the unrounded centroids are
    # not, for values close to a midpoint
    rng = np.random.default_rng(47)
    n_out, k_in, bits = 6, 4096, 3
    w = (rng.standard_normal((n_out, k_in)) * 0.02).astype(np.float16)
    r = orc.encode(w.view(np.uint16), bits, 0.0045, 30)
    dense = w.astype(np.float64).copy()
    for i in range(n_out):
        dense[i, r["col"][r["rowptr"][i]:r["rowptr"][i + 1]]] = 0.0
    for i in range(n_out):
        lut = r["lut"][i].view(np.float16).astype(np.float64)
        want = np.argmin(np.abs(dense[i][:, None] - lut[None, :]), axis=1)
        got = np.array(bigint_codes(r["codes"][i], bits, k_in))
        assert np.array_equal(got, want), (i, int((got != want).sum()))


def pin_enc_layer_reconstruction(orc):
    rng = np.random.default_rng(46)
    n_out, k_in, frac = 12, 64, 0.03
    for bits in (3, 4):
        w = (rng.standard_normal((n_out, k_in)) * 0.02).astype(np.float16)
        w[rng.integers(0, n_out, 5), rng.integers(0, k_in, 5)] = np.float16(0.7)
        r = orc.encode(w.view(np.uint16), bits, frac, 40)
        m = orc.outliers_per_tail(w.size, frac)
        rowptr, col, val = r["rowptr"], r["col"], r["val"]
        assert rowptr[0] == 0 and rowptr[-1] == 2 * m and np.all(np.diff(rowptr) >= 0)
        wv = w.view(np.uint16)
        outl = np.zeros((n_out, k_in), dtype=bool)
        for i in range(n_out):
            cs = col[rowptr[i]:rowptr[i + 1]]
            assert np.all(np.diff(cs) > 0)
            assert np.array_equal(val[rowptr[i]:rowptr[i + 1]], wv[i, cs])
            outl[i, cs] = True
        for i in range(n_out):
            lut = [Fraction(float(x)) for x in r["lut"][i].view(np.float16)]
            codes = bigint_codes(r["codes"][i], bits, k_in)
            for k in range(k_in):
                target = Fraction(0) if outl[i, k] else Fraction(float(w[i, k]))
                dist = [abs(target - e) for e in lut]
                assert codes[k] == dist.index(min(dist)), (bits, i, k)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
