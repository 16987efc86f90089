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

/* ======================================================================
 * Encoder: Dense-and-Sparse split and per-row 1-D k-means
 * ("SqueezeLLM: Dense-and-Sparse Quantization", summary page, section
 * "Sensitivity-Based Non-Uniform Quantization", Equation 1 and the
 * weighted k-means procedure without the sensitivity weights; section
 * "The Dense-and-Sparse Decomposition", W = D + S with percentile
 * thresholds).  Readings taken where the pages leave a step open:
 *   - the thresholds are order statistics of all N*K weights of the
 *     layer: with m = floor(fraction * N * K / 2 + 1/2) (at most N*K/2),
 *     the outliers are the first m and the last m weights in ascending
 *     order of (value, row-major position); D is W with those positions set
 *     to +0 and S holds them exactly (CSR, row-major, ascending column);
 *   - k-means runs per output row on the K values of that row of D (the
 *     zeros at outlier positions included), k = 2^b centroids initialised
 *     uniformly over [min, max] of the row (the uniform grid of the page);
 *   - one Lloyd iteration assigns every value to its nearest centroid
 *     (|d - c_j| in fp64, the lowest j on a tie) and sets each centroid to
 *     the mean of its values (sum in ascending column order, then one
 *     division); a centroid with no values keeps its place; iterations stop
 *     when no centroid moves or after max_iters;
 *   - the LUT holds the final centroids rounded to fp16 (to nearest, ties
 *     to even), and every weight's code is its nearest LUT entry (lowest
 *     index on a tie);
 *   - weights must be finite, and K * max|w| < 2^29 (every partial sum of a
 *     row's fp16 values is then exact in fp64).
 * ====================================================================== */
#include <stdlib.h>

/* double -> binary16, round to nearest, ties to even, from the format's
 * definition (overflow to infinity). */
uint16_t oracle_double_to_half(double v) {
    uint16_t sign = (uint16_t)(signbit(v) ? 0x8000u : 0u);
    double a = fabs(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00u);
    if (isinf(a)) return (uint16_t)(sign | 0x7c00u);
    /* largest finite half is 65504; values >= 65520 round to infinity */
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    int e;
    (void)frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;     /* a in [2^ex, 2^(ex+1)) */
    if (a == 0.0) return sign;
    if (ex < -14) ex = -14; /* subnormal range: quantum 2^-24 */
    double q = ldexp(1.0, ex - 10);  /* spacing of halves in this binade */
    double n = a / q;               /* exact: q is a power of two */
    double fl = floor(n);
    double r = n - fl;
    if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) == 1.0)) fl += 1.0;
    double rounded = fl * q;        /* exact */
    if (rounded >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    if (rounded < ldexp(1.0, -14)) {
        return (uint16_t)(sign | (uint16_t)(rounded / ldexp(1.0, -24))); /* subnormal: mantissa only */
    }
    int e2;
    double f2 = frexp(rounded, &e2); /* rounded = f2 * 2^e2 */
    int biased = e2 - 1 + 15;
    uint16_t mant = (uint16_t)((f2 * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)(biased << 10) | mant);
}

int64_t oracle_outliers_per_tail(int64_t n, double fraction) {
    if (n <= 0 || !(fraction >= 0.0)) return 0;
    int64_t m = (int64_t)floor(fraction * (double)n / 2.0 + 0.5);
    if (m > n / 2) m = n / 2;
    return m;
}

typedef struct {
    double v;
    int64_t pos;
} oracle_vp;

static int oracle_vp_cmp(const void* a, const void* b) {
    const oracle_vp* x = (const oracle_vp*)a;
    const oracle_vp* y = (const oracle_vp*)b;
    if (x->v < y->v) return -1;
    if (x->v > y->v) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos) ? 1 : 0;
}

/* marks[p] = 1 where weight p (row-major) is an outlier: the first m and the
 * last m in ascending (value, position) order. */
int oracle_select_outliers(int32_t n_out, int32_t k_in, const uint16_t* w, int64_t m, uint8_t* marks) {
    int64_t n = (int64_t)n_out * k_in;
    if (n_out < 0 || k_in < 0 || m < 0 || 2 * m > n) return ORACLE_BAD_ARG;
    memset(marks, 0, (size_t)n);
    if (m == 0) return ORACLE_OK;
    oracle_vp* a = (oracle_vp*)malloc((size_t)n * sizeof(oracle_vp));
    if (!a) return ORACLE_BAD_ARG;
    for (int64_t p = 0; p < n; ++p) {
        a[p].v = oracle_half_to_double(w[p]) + 0.0; /* -0 and +0 are one value */
        a[p].pos = p;
    }
    qsort(a, (size_t)n, sizeof(oracle_vp), oracle_vp_cmp);
    for (int64_t t = 0; t < m; ++t) {
        marks[a[t].pos] = 1;
        marks[a[n - 1 - t].pos] = 1;
    }
    free(a);
    return ORACLE_OK;
}

/* 1-D k-means (Lloyd) of n values, kc centroids; returns the iterations run. */
int oracle_kmeans_row(int64_t n, const double* d, int kc, int max_iters, double* c) {
    if (n <= 0 || kc < 2 || kc > 16) return -1;
    double lo = d[0], hi = d[0];
    for (int64_t k = 1; k < n; ++k) {
        if (d[k] < lo) lo = d[k];
        if (d[k] > hi) hi = d[k];
    }
    double step = (hi - lo) / (double)(kc - 1);
    for (int j = 0; j < kc; ++j) c[j] = lo + (double)j * step;
    int it = 0;
    for (; it < max_iters; ++it) {
        double sum[16];
        int64_t cnt[16];
        for (int j = 0; j < kc; ++j) {
            sum[j] = 0.0;
            cnt[j] = 0;
        }
        for (int64_t k = 0; k < n; ++k) {
            int best = 0;
            double bd = fabs(d[k] - c[0]);
            for (int j = 1; j < kc; ++j) {
                double dj = fabs(d[k] - c[j]);
                if (dj < bd) {
                    bd = dj;
                    best = j;
                }
            }
            sum[best] += d[k];
            cnt[best] += 1;
        }
        int moved = 0;
        for (int j = 0; j < kc; ++j) {
            double nc = cnt[j] ? sum[j] / (double)cnt[j] : c[j];
            if (nc != c[j]) moved = 1;
            c[j] = nc;
        }
        if (!moved) {
            ++it;
            break;
        }
    }
    return it;
}

/* Encode a layer: outliers to CSR (all rows), then for each requested row
 * (all rows when rows == NULL) the k-means LUT and the codes.  codes is
 * [n_rows][K*bits/32] canonical words, lut [n_rows][2^bits]; rowptr, col,
 * val describe S for all rows (nnz_cap entries available). */
int oracle_encode(int32_t n_out, int32_t k_in, int bits, const uint16_t* w, double fraction, int max_iters,
                  const int32_t* rows, int32_t n_rows, uint32_t* codes, uint16_t* lut, int32_t* rowptr, int32_t* col,
                  uint16_t* val, int64_t nnz_cap, int64_t* nnz_out, int32_t* iters_out) {
    int64_t wpr = oracle_words_per_row(k_in, bits);
    if (wpr < 0 || n_out < 1 || k_in < 1 || max_iters < 0) return ORACLE_BAD_ARG;
    int64_t n = (int64_t)n_out * k_in;
    double amax = 0.0;
    for (int64_t p = 0; p < n; ++p) {
        double v = oracle_half_to_double(w[p]);
        if (!isfinite(v)) return ORACLE_BAD_ARG;
        if (fabs(v) > amax) amax = fabs(v);
    }
    if (amax * (double)k_in >= ldexp(1.0, 29)) return ORACLE_BAD_ARG;
    int64_t m = oracle_outliers_per_tail(n, fraction);
    uint8_t* marks = (uint8_t*)malloc((size_t)n);
    if (!marks) return ORACLE_BAD_ARG;
    if (oracle_select_outliers(n_out, k_in, w, m, marks) != ORACLE_OK) {
        free(marks);
        return ORACLE_BAD_ARG;
    }
    int64_t nnz = 0;
    rowptr[0] = 0;
    for (int64_t i = 0; i < n_out; ++i) {
        for (int64_t k = 0; k < k_in; ++k) {
            if (!marks[i * k_in + k]) continue;
            if (nnz >= nnz_cap) {
                free(marks);
                return ORACLE_BAD_ARG;
            }
            col[nnz] = (int32_t)k;
            val[nnz] = w[i * k_in + k];
            ++nnz;
        }
        rowptr[i + 1] = (int32_t)nnz;
    }
    *nnz_out = nnz;
    int L = 1 << bits;
    if (rows == NULL) n_rows = n_out;
    double* d = (double*)malloc((size_t)k_in * sizeof(double));
    uint8_t* cm = (uint8_t*)malloc((size_t)k_in);
    if (!d || !cm) {
        free(marks);
        free(d);
        free(cm);
        return ORACLE_BAD_ARG;
    }
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= n_out) {
            free(marks);
            free(d);
            free(cm);
            return ORACLE_BAD_ARG;
        }
        for (int64_t k = 0; k < k_in; ++k)
            d[k] = marks[i * k_in + k] ? 0.0 : oracle_half_to_double(w[i * k_in + k]) + 0.0;
        double c[16];
        int it = oracle_kmeans_row(k_in, d, L, max_iters, c);
        if (iters_out) iters_out[r] = it;
        double lv[16];
        for (int j = 0; j < L; ++j) {
            lut[r * L + j] = oracle_double_to_half(c[j]);
            lv[j] = oracle_half_to_double(lut[r * L + j]);
        }
        for (int64_t k = 0; k < k_in; ++k) {
            int best = 0;
            double bd = fabs(d[k] - lv[0]);
            for (int j = 1; j < L; ++j) {
                double dj = fabs(d[k] - lv[j]);
                if (dj < bd) {
                    bd = dj;
                    best = j;
                }
            }
            cm[k] = (uint8_t)best;
        }
        if (oracle_pack(1, k_in, bits, cm, codes + r * wpr) != ORACLE_OK) {
            free(marks);
            free(d);
            free(cm);
            return ORACLE_BAD_ARG;
        }
    }
    free(marks);
    free(d);
    free(cm);
    return ORACLE_OK;
}
