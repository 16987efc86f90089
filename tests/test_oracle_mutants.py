"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pin battery catches every one of them."""
import os
import re
import shutil

import pytest

import oracle
from pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "sqz_oracle.c")

# (name, pattern, replacement): each is a mistake a transcription could make.
MUTANTS = [
    ("drop_sparse_term", r"ys \+= t;", "ys += 0.0 * t;"),
    ("sparse_sign", r"y\[b \* n_rows \+ r\] = yd \+ ys;", "y[b * n_rows + r] = yd - ys;"),
    ("bit_order_reversed", r"int64_t p = k \* bits \+ t;\n        uint32_t bit",
     "int64_t p = k * bits + (bits - 1 - t);\n        uint32_t bit"),
    ("x_row_stride_k", r"x \+ b \* ldx", "x + b * k_in"),
    ("lut_row_index", r"lut\[i \* L \+ oracle_code\(row_words", "lut[(i / 2) * L + oracle_code(row_words"),
    ("x_gather_by_position", r"xb\[col\[j\]\]", "xb[j % k_in]"),
    ("subnormal_exponent", r"ldexp\(\(double\)f, -24\)", "ldexp((double)f, -25)"),
    ("exponent_bias", r"e - 25\)", "e - 24)"),
    ("code_row_stride", r"codes \+ i \* wpr;\n        for \(int64_t b", "codes + (i % 2) * wpr;\n        for (int64_t b"),
    ("row_end_exclusive", r"j < rowptr\[i \+ 1\]; \+\+j\) \{\n                    double t",
     "j < rowptr[i + 1] - 1; ++j) {\n                    double t"),
    # encoder
    ("half_truncates", r"if \(r > 0\.5 \|\| \(r == 0\.5 && fmod\(fl, 2\.0\) == 1\.0\)\) fl \+= 1\.0;", ""),
    ("half_ties_up", r"r == 0\.5 && fmod\(fl, 2\.0\) == 1\.0", "r == 0.5"),
    ("one_tail_only", r"marks\[a\[n - 1 - t\]\.pos\] = 1;", ""),
    ("tail_rounding_floor", r"floor\(fraction \* \(double\)n / 2\.0 \+ 0\.5\)", "floor(fraction * (double)n / 2.0)"),
    ("ties_by_position_reversed", r"return \(x->pos < y->pos\) \? -1 : \(x->pos > y->pos\) \? 1 : 0;",
     "return (x->pos < y->pos) ? 1 : (x->pos > y->pos) ? -1 : 0;"),
    ("init_grid_from_zero", r"c\[j\] = lo \+ \(double\)j \* step;", "c[j] = (double)j * step;"),
    ("empty_cluster_to_zero", r"cnt\[j\] \? sum\[j\] / \(double\)cnt\[j\] : c\[j\]", "cnt[j] ? sum[j] / (double)cnt[j] : 0.0"),
    ("mean_over_all_values", r"sum\[j\] / \(double\)cnt\[j\]", "sum[j] / (double)n"),
    ("outliers_left_in_dense", r"d\[k\] = marks\[i \* k_in \+ k\] \? 0\.0 : ", "d[k] = marks[i * k_in + k] ? oracle_half_to_double(w[i * k_in + k]) : "),
    ("codes_from_unrounded_centroids", r"lv\[j\] = oracle_half_to_double\(lut\[r \* L \+ j\]\);", "lv[j] = c[j];"),
]


@pytest.mark.parametrize("name,pat,rep", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, pat, rep):
    src = open(SRC).read()
    mutated, n = re.subn(pat, rep, src)
    assert n >= 1, f"mutation {name} did not apply"
    csrc = tmp_path / "mut.c"
    csrc.write_text(mutated)
    lib_path = oracle.build(force=True, src=str(csrc), out=str(tmp_path / "libmut.so"))
    mut = oracle.Oracle(oracle.load(lib_path))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mut)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
