/*
 * sqz_oracle.c -- CPU oracle for the Dense-and-Sparse quantized GEMV.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * fp64 reference that the CUDA path is checked against.  It shares no code,
 * header, table or helper with the CUDA library; only the test suite, the
 * package's smoke check and the benchmark's CPU-baseline leg may load it.
 *
 * What it computes ("SqueezeLLM: Dense-and-Sparse Quantization", summary
 * page, §3.4 "The Dense-and-Sparse Decomposition" and "Kernel
 * Implementation"):
 *
 *     W = D + S,   y = W x = Q(D) x + S x
 *
 * where Q(D) stores every weight as a b-bit index into a per-output-row
 * lookup table of 2^b fp16 centroids (§3.2 "Sensitivity-Based K-Means
 * Quantizer", channel-wise LUTs) and S is an fp16 matrix in CSR form
 * (values, col_indices, row_ptr; §3.4 "The Sparse Matrix Storage Format").
 *
 * Readings taken where the pages are silent (each also listed in the
 * design notes):
 *   - codes of one row form one LSB-first bitstream of little-endian 32-bit
 *     words, K*b bits long, rows back to back with no padding (§3.4 "The 3/4-bit
 *     storage format": indices use exactly 3 or 4 bits, 8 three-bit indices
 *     in 3 bytes);
 *   - "per channel" is per output row;
 *   - Q and S are added: every (i,k) has a code, S is added on top;
 *   - CSR columns are int32, may be unsorted, duplicates are summed, empty
 *     rows are allowed;
 *   - summation order is not specified; this oracle sums in ascending k and
 *     ascending CSR position, in fp64.
 *
 * Every function is a direct transcription of a definition; there is no
 * blocking, fusion or reordering.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* IEEE 754 binary16 -> double, from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -24);               /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        mag = (f == 0) ? INFINITY : NAN;
    } else {
        mag = ldexp((double)(1024 + f), e - 25);    /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

static int bits_ok(int bits) { return bits == 3 || bits == 4; }

/* Number of 32-bit words holding one row: K*b bits, no padding. */
int64_t oracle_words_per_row(int64_t k_in, int bits) {
    if (!bits_ok(bits) || k_in < 0 || (k_in * bits) % 32 != 0) return -1;
    return k_in * bits / 32;
}

/* code(i,k): the b-bit field starting at bit k*b of row i's bitstream.
 * Bit p of the stream is bit (p mod 32) of word (p div 32).  A field may
 * straddle two words (3-bit codes 10 and 21 of every 96-bit group). */
uint32_t oracle_code(const uint32_t* row_words, int bits, int64_t k) {
    uint32_t code = 0;
    for (int t = 0; t < bits; ++t) {
        int64_t p = k * bits + t;
        uint32_t bit = (row_words[p / 32] >> (p % 32)) & 1u;
        code |= bit << t;
    }
    return code;
}

/* Unpack all codes: out[i*k_in + k] = code(i,k). */
int oracle_unpack(int32_t n_out, int32_t k_in, int bits, const uint32_t* codes, uint8_t* out) {
    int64_t wpr = oracle_words_per_row(k_in, bits);
    if (wpr < 0 || n_out < 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_out; ++i)
        for (int64_t k = 0; k < k_in; ++k)
            out[i * k_in + k] = (uint8_t)oracle_code(codes + i * wpr, bits, k);
    return ORACLE_OK;
}

/* Inverse of oracle_unpack: write each code's b bits at bit k*b of its row. */
int oracle_pack(int32_t n_out, int32_t k_in, int bits, const uint8_t* in, uint32_t* codes) {
    int64_t wpr = oracle_words_per_row(k_in, bits);
    if (wpr < 0 || n_out < 0) return ORACLE_BAD_ARG;
    memset(codes, 0, (size_t)(n_out * wpr) * sizeof(uint32_t));
    for (int64_t i = 0; i < n_out; ++i)
        for (int64_t k = 0; k < k_in; ++k) {
            uint32_t c = in[i * k_in + k];
            if (c >> bits) return ORACLE_BAD_ARG;
            for (int t = 0; t < bits; ++t) {
                int64_t p = k * bits + t;
                codes[i * wpr + p / 32] |= ((c >> t) & 1u) << (p % 32);
            }
        }
    return ORACLE_OK;
}

/* Dequantized dense weights: w(i,k) = lut[i][code(i,k)], as fp16 bit
 * patterns (a table lookup, no arithmetic). */
int oracle_dequant(int32_t n_out, int32_t k_in, int bits, const uint32_t* codes, const uint16_t* lut,
                   uint16_t* w_out) {
    int64_t wpr = oracle_words_per_row(k_in, bits);
    if (wpr < 0 || n_out < 0) return ORACLE_BAD_ARG;
    int64_t L = (int64_t)1 << bits;
    for (int64_t i = 0; i < n_out; ++i)
        for (int64_t k = 0; k < k_in; ++k)
            w_out[i * k_in + k] = lut[i * L + oracle_code(codes + i * wpr, bits, k)];
    return ORACLE_OK;
}

/* CSR well-formedness: row_ptr[0] = 0, non-decreasing, row_ptr[N] = nnz,
 * every column in [0, K).  Returns ORACLE_OK or ORACLE_BAD_ARG. */
int oracle_check_csr(int32_t n_out, int32_t k_in, int64_t nnz, const int32_t* rowptr, const int32_t* col) {
    if (nnz == 0 && rowptr == NULL) return ORACLE_OK;
    if (rowptr[0] != 0 || (int64_t)rowptr[n_out] != nnz) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_out; ++i)
        if (rowptr[i + 1] < rowptr[i]) return ORACLE_BAD_ARG;
    for (int64_t j = 0; j < nnz; ++j)
        if (col[j] < 0 || col[j] >= k_in) return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/*
 * y = (Q + S) x for the rows listed in `rows` (all rows when rows == NULL),
 * batch columns b = 0..batch-1.
 *
 *   yd(i,b) = sum_k lut[i][code(i,k)] * x[b][k]                (dense part)
 *   ys(i,b) = sum_{j=rowptr[i]}^{rowptr[i+1]-1} val[j] * x[b][col[j]]   (CSR)
 *   y(i,b)  = yd + ys
 *   bound(i,b) = sum_k |w(i,k) x[b][k]| + sum_j |val[j] x[b][col[j]]|
 *
 * Outputs are indexed [b][r] with r the position of the row in `rows`
 * (or the row itself when rows == NULL): y[b*n_rows + r].
 * nnz == 0 allows rowptr/col/val == NULL.
 */
int oracle_gemv(int32_t n_out, int32_t k_in, int bits, const uint32_t* codes, const uint16_t* lut,
                int64_t nnz, const int32_t* rowptr, const int32_t* col, const uint16_t* val,
                const uint16_t* x, int32_t batch, int64_t ldx,
                const int32_t* rows, int64_t n_rows, double* y, double* bound) {
    int64_t wpr = oracle_words_per_row(k_in, bits);
    if (wpr < 0 || n_out < 0 || batch < 0 || ldx < k_in) return ORACLE_BAD_ARG;
    if (oracle_check_csr(n_out, k_in, nnz, rowptr, col) != ORACLE_OK) return ORACLE_BAD_ARG;
    if (rows == NULL) n_rows = n_out;
    int64_t L = (int64_t)1 << bits;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= n_out) return ORACLE_BAD_ARG;
        const uint32_t* row_words = codes + i * wpr;
        for (int64_t b = 0; b < batch; ++b) {
            const uint16_t* xb = x + b * ldx;
            double yd = 0.0, ys = 0.0, bd = 0.0;
            for (int64_t k = 0; k < k_in; ++k) {
                double w = oracle_half_to_double(lut[i * L + oracle_code(row_words, bits, k)]);
                double t = w * oracle_half_to_double(xb[k]);
                yd += t;
                bd += fabs(t);
            }
            if (nnz > 0) {
                for (int64_t j = rowptr[i]; j < rowptr[i + 1]; ++j) {
                    double t = oracle_half_to_double(val[j]) * oracle_half_to_double(xb[col[j]]);
                    ys += t;
                    bd += fabs(t);
                }
            }
            y[b * n_rows + r] = yd + ys;
            if (bound) bound[b * n_rows + r] = bd;
        }
    }
    return ORACLE_OK;
}
