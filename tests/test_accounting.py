"""P-7: the byte accounting reproduces the average bits the pages print
(per-row LUTs, fp16 value + int32 column per outlier), and a 16-bit column
index does not."""
from pins import read_golden

from lut_dequant_gemv_b200 import accounting as acc


def test_avg_bits_match_printed_table():
    for bits, p, printed in ((int(a), float(b), float(c)) for a, b, c in read_golden("avg_bits_llama7b.txt")):
        got = acc.avg_bits(acc.LLAMA7B_LAYER, bits, p, bits_per_nnz=48)
        assert abs(got - printed) <= 0.01, (bits, p, got, printed)


def test_sixteen_bit_columns_do_not_match():
    for bits, p, printed in ((int(a), float(b), float(c)) for a, b, c in read_golden("avg_bits_llama7b.txt")):
        if p > 0:
            got = acc.avg_bits(acc.LLAMA7B_LAYER, bits, p, bits_per_nnz=32)
            assert abs(got - printed) > 0.05


def test_gemv_bytes_formula():
    # 11008 x 4096, 3-bit, 0.45 % outliers, batch 1
    n, k, nnz = 11008, 4096, 202899
    b = acc.gemv_bytes(n, k, 3, nnz, 1)
    assert b == n * k * 3 // 8 + n * 8 * 2 + 6 * nnz + 4 * (n + 1) + 2 * (k + n)
    assert acc.gemv_bytes(n, k, 3, 0, 1) == n * k * 3 // 8 + n * 16 + 2 * (k + n)
