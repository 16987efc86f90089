// sqz_encode.cu -- encoder: fp16 weights -> (codes, LUT, CSR outliers).
//
// Follows "SqueezeLLM: Dense-and-Sparse Quantization" (summary page):
// section "The Dense-and-Sparse Decomposition" (W = D + S, S the weights
// beyond percentile thresholds, kept exactly) and section
// "Sensitivity-Based Non-Uniform Quantization" (Eq. 1: per output row, a
// 1-D k-means over the row's values gives 2^b centroids -- the row's fp16
// LUT -- and every weight is stored as the index of its centroid), without
// the sensitivity weights.  The steps the pages leave open are fixed so
// that every decision is exact and independent of scheduling:
//   - outliers: with m = floor(fraction * N * K / 2 + 1/2) (at most half),
//     the first m and the last m weights in ascending (value, row-major
//     position) order; -0 and +0 are one value.  Found by a two-level radix
//     count over 16-bit order keys and ranks of the threshold ties taken in
//     position order;
//   - D is W with the outliers set to +0; k-means per row of D from the
//     uniform grid over [min, max] of the row, Lloyd iterations (nearest
//     centroid by |d - c_j| in fp64, lowest j on a tie; each centroid the
//     mean of its values, an empty one keeps its place) until no centroid
//     moves or max_iters;
//   - a row's values are fp16, so their sums are integers in units of
//     2^-24: summed as 64-bit integers they are exact in any order, and the
//     mean is one fp64 division (this needs K * max|w| < 2^29);
//   - LUT = centroids rounded to fp16 (nearest, ties to even); code = the
//     nearest LUT entry (lowest index on a tie); codes in the canonical
//     LSB-first bitstream.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/sqz.h"

void sqz_internal_set_last_error(const char* msg);

namespace sqz {
namespace enc {

constexpr int kThreads = 256;
constexpr int kChunkBlocksMax = 4096;

// 16-bit key that orders fp16 values as numbers (-0 and +0 share one key;
// NaN is rejected before any key is formed).
__device__ __forceinline__ uint32_t order_key(uint16_t h) {
    if (h == 0x8000u) h = 0;
    return (h & 0x8000u) ? (~(uint32_t)h & 0xffffu) : ((uint32_t)h | 0x8000u);
}

// Non-finite weights (flag bit 0) and the largest magnitude (as the bits of
// a non-negative float, which order like the values).
__global__ void scan_kernel(const uint16_t* __restrict__ w, int64_t n, unsigned* __restrict__ amax_bits,
                            int* __restrict__ flag) {
    unsigned m = 0;
    int bad = 0;
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
        const uint16_t h = w[p];
        if ((h & 0x7c00u) == 0x7c00u) bad = 1;
        const float a = fabsf(__half2float(__ushort_as_half(h)));
        m = max(m, __float_as_uint(a));
    }
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, m);
    if (bad) atomicOr(flag, 1);
}

// Counts of the high byte of the key (sel < 0), or of the low byte among
// keys whose high byte is sel_a (hist_a) or sel_b (hist_b).
__global__ void hist_kernel(const uint16_t* __restrict__ w, int64_t n, int sel_a, int sel_b,
                            unsigned long long* __restrict__ hist_a, unsigned long long* __restrict__ hist_b) {
    __shared__ unsigned sa[256], sb[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sa[i] = sb[i] = 0;
    __syncthreads();
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t k = order_key(w[p]);
        if (sel_a < 0) {
            atomicAdd(&sa[k >> 8], 1u);
        } else {
            if ((int)(k >> 8) == sel_a) atomicAdd(&sa[k & 0xffu], 1u);
            if ((int)(k >> 8) == sel_b) atomicAdd(&sb[k & 0xffu], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        if (sa[i]) atomicAdd(&hist_a[i], (unsigned long long)sa[i]);
        if (sel_a >= 0 && sb[i]) atomicAdd(&hist_b[i], (unsigned long long)sb[i]);
    }
}

// Elements with key == key_lo / key_hi in each block's contiguous chunk.
__global__ void tie_count_kernel(const uint16_t* __restrict__ w, int64_t n, int64_t chunk, uint32_t key_lo,
                                 uint32_t key_hi, long long* __restrict__ cnt_lo, long long* __restrict__ cnt_hi) {
    const int64_t a = (int64_t)blockIdx.x * chunk, b = min(n, a + chunk);
    int lo = 0, hi = 0;
    for (int64_t p = a + threadIdx.x; p < b; p += blockDim.x) {
        const uint32_t k = order_key(w[p]);
        lo += k == key_lo;
        hi += k == key_hi;
    }
    for (int o = 16; o; o >>= 1) {
        lo += __shfl_xor_sync(0xffffffffu, lo, o);
        hi += __shfl_xor_sync(0xffffffffu, hi, o);
    }
    __shared__ int s_lo[kThreads / 32], s_hi[kThreads / 32];
    if ((threadIdx.x & 31) == 0) {
        s_lo[threadIdx.x >> 5] = lo;
        s_hi[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        long long tl = 0, th = 0;
        for (int i = 0; i < kThreads / 32; ++i) tl += s_lo[i], th += s_hi[i];
        cnt_lo[blockIdx.x] = tl;
        cnt_hi[blockIdx.x] = th;
    }
}

// Rank (in position order) among the elements of this block's chunk that
// satisfy `pred`, for the element the calling thread holds this round;
// `running` carries the count of earlier rounds.  All threads of the block
// call it together.
__device__ __forceinline__ long long ordered_rank(bool pred, long long& running, int* s_warp) {
    const unsigned bal = __ballot_sync(0xffffffffu, pred);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int before = __popc(bal & ((1u << lane) - 1u));
    __syncthreads();
    if (lane == 0) s_warp[wid] = __popc(bal);
    __syncthreads();
    int warp_off = 0, total = 0;
    for (int i = 0; i < kThreads / 32; ++i) {
        warp_off += i < wid ? s_warp[i] : 0;
        total += s_warp[i];
    }
    const long long r = running + warp_off + before;
    running += total;
    return r;
}

// flags[p] = 1 for the outliers: keys below key_lo or above key_hi, the
// first r_lo elements with key == key_lo and the last r_hi with key ==
// key_hi (position order; tie_hi elements have key == key_hi in all).
__global__ void __launch_bounds__(kThreads) mark_kernel(const uint16_t* __restrict__ w, int64_t n, int64_t chunk,
                                                        uint32_t key_lo, uint32_t key_hi,
                                                        const long long* __restrict__ pre_lo,
                                                        const long long* __restrict__ pre_hi, long long r_lo,
                                                        long long r_hi, long long tie_hi, uint8_t* __restrict__ flags) {
    __shared__ int s_warp[kThreads / 32];
    const int64_t a = (int64_t)blockIdx.x * chunk, b = min(n, a + chunk);
    long long run_lo = pre_lo[blockIdx.x], run_hi = pre_hi[blockIdx.x];
    for (int64_t base = a; base < b; base += kThreads) {
        const int64_t p = base + threadIdx.x;
        const bool in = p < b;
        const uint32_t k = in ? order_key(w[p]) : 0u;
        const bool eq_lo = in && k == key_lo, eq_hi = in && k == key_hi;
        const long long rk_lo = ordered_rank(eq_lo, run_lo, s_warp);
        const long long rk_hi = ordered_rank(eq_hi, run_hi, s_warp);
        if (in) {
            const bool out = k < key_lo || k > key_hi || (eq_lo && rk_lo < r_lo) || (eq_hi && rk_hi >= tie_hi - r_hi);
            flags[p] = out ? 1 : 0;
        }
    }
}

// Outliers per row (one warp per row).
__global__ void row_count_kernel(const uint8_t* __restrict__ flags, int32_t n_out, int32_t k_in,
                                 int* __restrict__ counts) {
    const int lane = threadIdx.x & 31;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n_out;
         i += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        int c = 0;
        for (int64_t k = lane; k < k_in; k += 32) c += flags[i * k_in + k];
        for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) counts[i] = c;
    }
}

// S in CSR: the row's outliers in ascending column order (one warp per row).
__global__ void csr_fill_kernel(const uint16_t* __restrict__ w, const uint8_t* __restrict__ flags, int32_t n_out,
                                int32_t k_in, const int32_t* __restrict__ rowptr, int32_t* __restrict__ col,
                                uint16_t* __restrict__ val) {
    const int lane = threadIdx.x & 31;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n_out;
         i += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        int pos = rowptr[i];
        for (int64_t k0 = 0; k0 < k_in; k0 += 32) {
            const int64_t k = k0 + lane;
            const bool f = k < k_in && flags[i * k_in + k];
            const unsigned bal = __ballot_sync(0xffffffffu, f);
            if (f) {
                const int at = pos + __popc(bal & ((1u << lane) - 1u));
                col[at] = (int32_t)k;
                val[at] = w[i * k_in + k];
            }
            pos += __popc(bal);
        }
    }
}

// fp64 -> fp16 bits, round to nearest, ties to even (from the binary16
// format: 1 sign, 5 exponent bits with bias 15, 10 fraction bits).
__device__ __forceinline__ uint16_t d2h_rne(double v) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(v);
    const uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    const int e = (int)((b >> 52) & 0x7ff);
    const unsigned long long frac = b & ((1ull << 52) - 1);
    if (e == 0x7ff) return (uint16_t)(sign | (frac ? 0x7e00u : 0x7c00u));
    if (e == 0) return sign;  // double zero or subnormal: far below the smallest half
    const int ue = e - 1023;
    if (ue > 15) return (uint16_t)(sign | 0x7c00u);
    const unsigned long long sig = frac | (1ull << 52);
    const int shift = ue >= -14 ? 42 : 42 + (-14 - ue);
    if (shift > 60) return sign;
    unsigned long long q = sig >> shift;
    const unsigned long long rem = sig & ((1ull << shift) - 1), halfway = 1ull << (shift - 1);
    if (rem > halfway || (rem == halfway && (q & 1))) ++q;
    if (ue >= -14) {
        int he = ue + 15;
        if (q == 2048) {
            q = 1024;
            ++he;
        }
        if (he >= 31) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | (he << 10) | (uint16_t)(q - 1024));
    }
    return (uint16_t)(sign | (uint16_t)q);  // subnormal (q == 1024 is the smallest normal)
}

// One CTA of kThreads threads per row: Lloyd k-means on the row of D, then
// the LUT and the codes.  The row of D is first copied into shared memory
// (fp16, +0 at the outliers and for -0); each iteration every thread
// assigns its values (columns tid, tid + kThreads, ...) and sums them per
// centroid as integers in units of 2^-24, the warps' sums are added in
// shared memory (integer sums: exact in any order), and the new centroids
// are formed once and broadcast.
template <int BITS>
__global__ void __launch_bounds__(kThreads) kmeans_kernel(const uint16_t* __restrict__ w,
                                                          const uint8_t* __restrict__ flags, int32_t n_out,
                                                          int32_t k_in, int max_iters, uint32_t* __restrict__ codes,
                                                          uint16_t* __restrict__ lut, int32_t* __restrict__ iters_out) {
    constexpr int L = 1 << BITS;
    constexpr int NW = kThreads / 32;
    extern __shared__ __align__(16) uint16_t dr[];  // [k_in]
    __shared__ long long s_sum[NW][L];
    __shared__ int s_cnt[NW][L];
    __shared__ double s_c[L], s_lo[NW], s_hi[NW];
    __shared__ int s_moved;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t wpr = (int64_t)k_in * BITS / 32;
    for (int64_t i = blockIdx.x; i < n_out; i += gridDim.x) {
        const uint16_t* wr = w + i * k_in;
        const uint8_t* fr = flags + i * k_in;
        __syncthreads();
        double lo = INFINITY, hi = -INFINITY;
        for (int64_t k = tid; k < k_in; k += kThreads) {
            const uint16_t h = wr[k];
            const uint16_t v = (fr[k] || h == 0x8000u) ? (uint16_t)0 : h;
            dr[k] = v;
            const double d = (double)__half2float(__ushort_as_half(v));
            lo = fmin(lo, d);
            hi = fmax(hi, d);
        }
        for (int o = 16; o; o >>= 1) {
            lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (lane == 0) {
            s_lo[wid] = lo;
            s_hi[wid] = hi;
        }
        __syncthreads();
        lo = s_lo[0];
        hi = s_hi[0];
#pragma unroll
        for (int v = 1; v < NW; ++v) {
            lo = fmin(lo, s_lo[v]);
            hi = fmax(hi, s_hi[v]);
        }
        double c[L];
        const double step = __ddiv_rn(__dsub_rn(hi, lo), (double)(L - 1));
#pragma unroll
        for (int j = 0; j < L; ++j) c[j] = __dadd_rn(lo, __dmul_rn((double)j, step));
        int it = 0;
        for (; it < max_iters; ++it) {
            long long sm[L];
            int cnt[L];
#pragma unroll
            for (int j = 0; j < L; ++j) sm[j] = 0, cnt[j] = 0;
            for (int64_t k = tid; k < k_in; k += kThreads) {
                const double d = (double)__half2float(__ushort_as_half(dr[k]));
                const long long di = __double2ll_rn(__dmul_rn(d, 16777216.0));  // exact: d is a multiple of 2^-24
                int best = 0;
                double bd = fabs(__dsub_rn(d, c[0]));
#pragma unroll
                for (int j = 1; j < L; ++j) {
                    const double dj = fabs(__dsub_rn(d, c[j]));
                    if (dj < bd) {
                        bd = dj;
                        best = j;
                    }
                }
#pragma unroll
                for (int j = 0; j < L; ++j)
                    if (best == j) {
                        sm[j] += di;
                        cnt[j] += 1;
                    }
            }
#pragma unroll
            for (int j = 0; j < L; ++j) {
                for (int o = 16; o; o >>= 1) {
                    sm[j] += __shfl_xor_sync(0xffffffffu, sm[j], o);
                    cnt[j] += __shfl_xor_sync(0xffffffffu, cnt[j], o);
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < L; ++j) {
                    s_sum[wid][j] = sm[j];
                    s_cnt[wid][j] = cnt[j];
                }
            }
            if (tid == 0) s_moved = 0;
            __syncthreads();
            if (tid < L) {
                long long tot = 0;
                int n = 0;
#pragma unroll
                for (int v = 0; v < NW; ++v) {
                    tot += s_sum[v][tid];
                    n += s_cnt[v][tid];
                }
                double cj = 0.0;
#pragma unroll
                for (int j = 0; j < L; ++j)
                    if (j == tid) cj = c[j];
                const double nc = n ? __ddiv_rn(__dmul_rn((double)tot, 0x1p-24), (double)n) : cj;
                if (nc != cj) s_moved = 1;
                s_c[tid] = nc;
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < L; ++j) c[j] = s_c[j];
            const bool moved = s_moved != 0;
            __syncthreads();  // s_moved and the sums are rewritten next iteration
            if (!moved) {
                ++it;
                break;
            }
        }
        if (iters_out && tid == 0) iters_out[i] = it;
        // the LUT and each weight's nearest entry
        double lv[L];
#pragma unroll
        for (int j = 0; j < L; ++j) {
            const uint16_t hb = d2h_rne(c[j]);
            lv[j] = (double)__half2float(__ushort_as_half(hb));
            if (tid == j) lut[i * L + j] = hb;
        }
        uint32_t* cw = codes + i * wpr;
        for (int64_t k0 = (int64_t)wid * 32; k0 < k_in; k0 += kThreads) {
            const int64_t k = k0 + lane;
            uint32_t code = 0;
            if (k < k_in) {
                const double d = (double)__half2float(__ushort_as_half(dr[k]));
                double bd = fabs(__dsub_rn(d, lv[0]));
#pragma unroll
                for (int j = 1; j < L; ++j) {
                    const double dj = fabs(__dsub_rn(d, lv[j]));
                    if (dj < bd) {
                        bd = dj;
                        code = (uint32_t)j;
                    }
                }
            }
            // the 32 codes of this group occupy BITS words starting at word k0*BITS/32
            const int t = lane * BITS;  // bit offset of this lane's code in the group
#pragma unroll
            for (int q = 0; q < BITS; ++q) {
                uint32_t part = 0;
                const int lo_bit = t - 32 * q;  // position of the code's bit 0 within word q
                if (lo_bit >= 0 && lo_bit < 32) part = code << lo_bit;
                else if (lo_bit < 0 && lo_bit > -BITS) part = code >> (-lo_bit);
                const uint32_t word = __reduce_or_sync(0xffffffffu, part);
                const int64_t wi = k0 * BITS / 32 + q;
                if (lane == 0 && wi < wpr) cw[wi] = word;
            }
        }
    }
}

}  // namespace enc
}  // namespace sqz

namespace {

sqz_status enc_fail(sqz_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    sqz_internal_set_last_error(buf);
    return st;
}

// Device workspace of one encode call, released on every return path.
struct Workspace {
    std::vector<void*> ptrs;
    ~Workspace() {
        for (void* p : ptrs) cudaFree(p);
    }
    template <class T>
    cudaError_t get(T** out, size_t count) {
        *out = nullptr;
        void* p = nullptr;
        cudaError_t e = cudaMalloc(&p, count * sizeof(T) > 0 ? count * sizeof(T) : 16);
        if (e == cudaSuccess) {
            ptrs.push_back(p);
            *out = static_cast<T*>(p);
        }
        return e;
    }
};

#define ENC_TRY(expr, what)                                                                                 \
    do {                                                                                                    \
        cudaError_t e_ = (expr);                                                                            \
        if (e_ != cudaSuccess) {                                                                            \
            (void)cudaGetLastError();                                                                       \
            return enc_fail(e_ == cudaErrorMemoryAllocation ? SQZ_ERR_OOM : SQZ_ERR_CUDA, "%s: %s (%s)", what, \
                            cudaGetErrorName(e_), cudaGetErrorString(e_));                                  \
        }                                                                                                   \
    } while (0)

int64_t per_tail(int64_t n, double fraction) {
    if (n <= 0 || !(fraction >= 0.0)) return 0;
    int64_t m = (int64_t)std::floor(fraction * (double)n / 2.0 + 0.5);
    return m > n / 2 ? n / 2 : m;
}

int grid_for(int64_t items, int per_block) {
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t g = (items + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sms * 16;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

extern "C" {

SQZ_API int64_t sqz_encode_outliers(int64_t n_weights, double fraction) { return 2 * per_tail(n_weights, fraction); }

SQZ_API sqz_status sqz_encode(const uint16_t* w, int32_t n_out, int32_t k_in, int32_t bits, double outlier_fraction,
                              int32_t max_iters, uint32_t* codes, uint16_t* lut, int32_t* rowptr, int32_t* col,
                              uint16_t* val, int64_t nnz_capacity, int64_t* nnz_out, int32_t* iters_out,
                              void* stream) {
    using namespace sqz::enc;
    if (nnz_out) *nnz_out = 0;
    if (!w || !codes || !lut || !rowptr || !nnz_out)
        return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: w, codes, lut, rowptr and nnz_out must be non-NULL");
    if (bits != 3 && bits != 4) return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: bits must be 3 or 4 (got %d)", bits);
    if (n_out < 1 || k_in < 1) return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: n_out and k_in must be positive");
    if (k_in % (bits == 3 ? 32 : 8) != 0)
        return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: k_in must be a multiple of %d for %d-bit codes",
                        bits == 3 ? 32 : 8, bits);
    if (!(outlier_fraction >= 0.0 && outlier_fraction <= 1.0))
        return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: outlier_fraction must lie in [0, 1]");
    if (max_iters < 0 || max_iters > 100000)
        return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: max_iters must lie in [0, 100000]");
    const int64_t n = (int64_t)n_out * k_in;
    const int64_t m = per_tail(n, outlier_fraction);
    if (2 * m > nnz_capacity)
        return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: %lld outliers need col/val of that many entries (capacity %lld)",
                        (long long)(2 * m), (long long)nnz_capacity);
    if (2 * m > 0 && (!col || !val)) return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: col and val must be non-NULL");
    if (2 * m > INT32_MAX - 64) return enc_fail(SQZ_ERR_UNSUPPORTED, "sqz_encode: too many outliers for int32 rowptr");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Workspace ws;

    // ---- finite weights, and K * max|w| < 2^29 (exact integer sums per row)
    unsigned* d_amax;
    int* d_flag;
    ENC_TRY(ws.get(&d_amax, 1), "encode workspace");
    ENC_TRY(ws.get(&d_flag, 1), "encode workspace");
    ENC_TRY(cudaMemsetAsync(d_amax, 0, sizeof(unsigned), s), "memset");
    ENC_TRY(cudaMemsetAsync(d_flag, 0, sizeof(int), s), "memset");
    scan_kernel<<<grid_for(n, kThreads), kThreads, 0, s>>>(w, n, d_amax, d_flag);
    ENC_TRY(cudaGetLastError(), "encode scan");
    unsigned h_amax = 0;
    int h_flag = 0;
    ENC_TRY(cudaMemcpyAsync(&h_amax, d_amax, sizeof h_amax, cudaMemcpyDeviceToHost, s), "copy");
    ENC_TRY(cudaMemcpyAsync(&h_flag, d_flag, sizeof h_flag, cudaMemcpyDeviceToHost, s), "copy");
    ENC_TRY(cudaStreamSynchronize(s), "encode scan");
    if (h_flag) return enc_fail(SQZ_ERR_INVALID_ARG, "sqz_encode: the weights contain inf or NaN");
    float amax;
    std::memcpy(&amax, &h_amax, sizeof amax);
    if ((double)amax * (double)k_in >= std::ldexp(1.0, 29))
        return enc_fail(SQZ_ERR_UNSUPPORTED, "sqz_encode: K * max|w| = %g reaches 2^29 (row sums no longer exact)",
                        (double)amax * (double)k_in);

    // ---- outlier flags
    uint8_t* d_flags;
    ENC_TRY(ws.get(&d_flags, (size_t)n), "encode workspace");
    if (m == 0) {
        ENC_TRY(cudaMemsetAsync(d_flags, 0, (size_t)n, s), "memset");
    } else {
        unsigned long long *d_ha, *d_hb;
        ENC_TRY(ws.get(&d_ha, 256), "encode workspace");
        ENC_TRY(ws.get(&d_hb, 256), "encode workspace");
        std::vector<unsigned long long> hh(256), hl(256), hr(256);
        ENC_TRY(cudaMemsetAsync(d_ha, 0, 256 * sizeof(unsigned long long), s), "memset");
        hist_kernel<<<grid_for(n, kThreads), kThreads, 0, s>>>(w, n, -1, -1, d_ha, d_hb);
        ENC_TRY(cudaGetLastError(), "encode histogram");
        ENC_TRY(cudaMemcpyAsync(hh.data(), d_ha, 256 * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s), "copy");
        ENC_TRY(cudaStreamSynchronize(s), "encode histogram");
        // high bytes holding the m-th smallest and the m-th largest key
        int blo = 0, bhi = 255;
        long long below = 0, above = 0;
        while ((long long)(below + hh[blo]) < m) below += hh[blo++];
        while ((long long)(above + hh[bhi]) < m) above += hh[bhi--];
        ENC_TRY(cudaMemsetAsync(d_ha, 0, 256 * sizeof(unsigned long long), s), "memset");
        ENC_TRY(cudaMemsetAsync(d_hb, 0, 256 * sizeof(unsigned long long), s), "memset");
        hist_kernel<<<grid_for(n, kThreads), kThreads, 0, s>>>(w, n, blo, bhi, d_ha, d_hb);
        ENC_TRY(cudaGetLastError(), "encode histogram");
        ENC_TRY(cudaMemcpyAsync(hl.data(), d_ha, 256 * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s), "copy");
        ENC_TRY(cudaMemcpyAsync(hr.data(), d_hb, 256 * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s), "copy");
        ENC_TRY(cudaStreamSynchronize(s), "encode histogram");
        int llo = 0, lhi = 255;
        while ((long long)(below + hl[llo]) < m) below += hl[llo++];
        while ((long long)(above + hr[lhi]) < m) above += hr[lhi--];
        const uint32_t key_lo = (uint32_t)(blo << 8 | llo), key_hi = (uint32_t)(bhi << 8 | lhi);
        const long long r_lo = m - below, r_hi = m - above, tie_hi = (long long)hr[lhi];
        // ranks of the threshold ties in position order: per-chunk counts, prefix on the host
        const int nb = (int)std::min<int64_t>(kChunkBlocksMax, (n + kThreads * 16 - 1) / (kThreads * 16));
        const int64_t chunk = ((n + nb - 1) / nb + kThreads - 1) / kThreads * kThreads;
        long long *d_cl, *d_ch;
        ENC_TRY(ws.get(&d_cl, nb), "encode workspace");
        ENC_TRY(ws.get(&d_ch, nb), "encode workspace");
        tie_count_kernel<<<nb, kThreads, 0, s>>>(w, n, chunk, key_lo, key_hi, d_cl, d_ch);
        ENC_TRY(cudaGetLastError(), "encode ties");
        std::vector<long long> cl(nb), ch(nb);
        ENC_TRY(cudaMemcpyAsync(cl.data(), d_cl, nb * sizeof(long long), cudaMemcpyDeviceToHost, s), "copy");
        ENC_TRY(cudaMemcpyAsync(ch.data(), d_ch, nb * sizeof(long long), cudaMemcpyDeviceToHost, s), "copy");
        ENC_TRY(cudaStreamSynchronize(s), "encode ties");
        long long al = 0, ah = 0;
        for (int b = 0; b < nb; ++b) {
            const long long tl = cl[b], th = ch[b];
            cl[b] = al;
            ch[b] = ah;
            al += tl;
            ah += th;
        }
        ENC_TRY(cudaMemcpyAsync(d_cl, cl.data(), nb * sizeof(long long), cudaMemcpyHostToDevice, s), "copy");
        ENC_TRY(cudaMemcpyAsync(d_ch, ch.data(), nb * sizeof(long long), cudaMemcpyHostToDevice, s), "copy");
        mark_kernel<<<nb, kThreads, 0, s>>>(w, n, chunk, key_lo, key_hi, d_cl, d_ch, r_lo, r_hi, tie_hi, d_flags);
        ENC_TRY(cudaGetLastError(), "encode marks");
        ENC_TRY(cudaStreamSynchronize(s), "encode marks");  // the host vectors above go out of scope
    }

    // ---- S in CSR
    int* d_counts;
    ENC_TRY(ws.get(&d_counts, (size_t)n_out), "encode workspace");
    const int warp_blocks = grid_for((int64_t)n_out * 32, kThreads);
    row_count_kernel<<<warp_blocks, kThreads, 0, s>>>(d_flags, n_out, k_in, d_counts);
    ENC_TRY(cudaGetLastError(), "encode row counts");
    std::vector<int32_t> rp((size_t)n_out + 1);
    ENC_TRY(cudaMemcpyAsync(rp.data() + 1, d_counts, sizeof(int32_t) * n_out, cudaMemcpyDeviceToHost, s), "copy");
    ENC_TRY(cudaStreamSynchronize(s), "encode row counts");
    rp[0] = 0;
    for (int32_t i = 0; i < n_out; ++i) rp[i + 1] += rp[i];
    if ((int64_t)rp[n_out] != 2 * m)
        return enc_fail(SQZ_ERR_CUDA, "sqz_encode: %d outliers marked, %lld expected", rp[n_out], (long long)(2 * m));
    ENC_TRY(cudaMemcpyAsync(rowptr, rp.data(), sizeof(int32_t) * ((size_t)n_out + 1), cudaMemcpyHostToDevice, s),
            "copy rowptr");
    if (m > 0) {
        csr_fill_kernel<<<warp_blocks, kThreads, 0, s>>>(w, d_flags, n_out, k_in, rowptr, col, val);
        ENC_TRY(cudaGetLastError(), "encode CSR");
    }

    // ---- k-means per row, LUT and codes (one CTA per row, the row in shared memory)
    const size_t smem = (size_t)k_in * 2;
    if (smem > 200u * 1024u)
        return enc_fail(SQZ_ERR_UNSUPPORTED, "sqz_encode: k_in = %d exceeds the %u columns a row stage holds", k_in,
                        (200u * 1024u) / 2u);
    const int kblocks = (int)std::min<int64_t>(n_out, 1 << 20);
    if (bits == 3) {
        ENC_TRY(cudaFuncSetAttribute(kmeans_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "encode attributes");
        kmeans_kernel<3><<<kblocks, kThreads, smem, s>>>(w, d_flags, n_out, k_in, max_iters, codes, lut, iters_out);
    } else {
        ENC_TRY(cudaFuncSetAttribute(kmeans_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "encode attributes");
        kmeans_kernel<4><<<kblocks, kThreads, smem, s>>>(w, d_flags, n_out, k_in, max_iters, codes, lut, iters_out);
    }
    ENC_TRY(cudaGetLastError(), "encode k-means");
    ENC_TRY(cudaStreamSynchronize(s), "encode k-means");
    *nnz_out = 2 * m;
    return SQZ_OK;
}

}  // extern "C"
