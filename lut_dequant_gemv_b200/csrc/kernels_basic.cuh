// kernels_basic.cuh -- CSR validation, dequant export and the row-per-warp
// fused GEMV over the canonical code layout.
//
// The fused GEMV follows "SqueezeLLM: Dense-and-Sparse Quantization"
// (summary page, §3.4 "Kernel Implementation"): codes are streamed from
// global memory, each is looked up in its row's LUT held on chip, the
// products with x are accumulated, the row's CSR outliers are added in the
// same kernel and y is written once.  The CSR part of a row is split evenly
// over the 32 lanes of the warp that owns the row (balanced within the row)
// and the lanes' partial sums are combined by one warp reduction, the same
// one that combines the dense partial sums -- no atomics.
#pragma once

#include "common.cuh"

namespace sqz {

// ---------------------------------------------------------------- CSR check
// Sets bits of *flag: 1 rowptr[0] != 0, 2 rowptr[N] != nnz, 4 rowptr
// decreasing, 8 column outside [0, K).  Internal linkage: every
// translation unit that launches it gets its own copy.
static __global__ void validate_csr_kernel(const int32_t* __restrict__ rowptr, const int32_t* __restrict__ col,
                                    int32_t n_out, int32_t k_in, int64_t nnz, int* __restrict__ flag) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int bad = 0;
    for (int64_t i = t0; i <= n_out; i += stride) {
        const int32_t r = rowptr[i];
        if (i == 0 && r != 0) bad |= 1;
        if (i == n_out && (int64_t)r != nnz) bad |= 2;
        if (i < n_out && rowptr[i + 1] < r) bad |= 4;
    }
    for (int64_t j = t0; j < nnz; j += stride) {
        const int32_t c = col[j];
        if (c < 0 || c >= k_in) bad |= 8;
    }
    if (bad) atomicOr(flag, bad);
}

// ------------------------------------------------------- canonical decoding
// Code j (0..31) of a 3-word, 32-code group of a 3-bit row: bits 3j..3j+2 of
// the 96-bit little-endian integer w0 + w1*2^32 + w2*2^64.
template <int J>
__device__ __forceinline__ uint32_t code3(uint32_t w0, uint32_t w1, uint32_t w2) {
    constexpr int p = 3 * J;
    if constexpr (p + 3 <= 32) {
        return (w0 >> p) & 7u;
    } else if constexpr (p < 32) {
        return ((w0 >> p) | (w1 << (32 - p))) & 7u;
    } else if constexpr (p + 3 <= 64) {
        return (w1 >> (p - 32)) & 7u;
    } else if constexpr (p < 64) {
        return ((w1 >> (p - 32)) | (w2 << (64 - p))) & 7u;
    } else {
        return (w2 >> (p - 64)) & 7u;
    }
}

template <int J, int BITS>
struct Unroll3 {
    template <class F>
    __device__ __forceinline__ static void run(uint32_t w0, uint32_t w1, uint32_t w2, F&& f) {
        f(J, code3<J>(w0, w1, w2));
        Unroll3<J + 1, BITS>::run(w0, w1, w2, f);
    }
};
template <int BITS>
struct Unroll3<32, BITS> {
    template <class F>
    __device__ __forceinline__ static void run(uint32_t, uint32_t, uint32_t, F&&) {}
};

// ------------------------------------------------------------ dequant export
// w_out[i][k] = lut[i][code(i,k)] from the canonical layout.
template <int BITS>
__global__ void dequant_canonical_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ lut,
                                         int32_t n_out, int32_t k_in, uint16_t* __restrict__ w_out) {
    constexpr int L = 1 << BITS;
    const int64_t wpr = (int64_t)k_in * BITS / 32;
    const int64_t units = (BITS == 3) ? k_in / 32 : wpr;  // 32 codes (3 words) or 8 codes (1 word)
    const int64_t total = (int64_t)n_out * units;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = t / units, u = t % units;
        const uint32_t* rw = codes + i * wpr;
        const uint16_t* lr = lut + i * L;
        uint16_t* out = w_out + i * k_in;
        if constexpr (BITS == 4) {
            const uint32_t w = rw[u];
#pragma unroll
            for (int j = 0; j < 8; ++j) out[u * 8 + j] = lr[(w >> (4 * j)) & 15u];
        } else {
            const uint32_t w0 = rw[3 * u], w1 = rw[3 * u + 1], w2 = rw[3 * u + 2];
            Unroll3<0, 3>::run(w0, w1, w2, [&](int j, uint32_t c) { out[u * 32 + j] = lr[c]; });
        }
    }
}

// ------------------------------------------------------- row-per-warp GEMV
// One warp per output row; the row's LUT is expanded to fp32 in shared
// memory (at most 16 entries, one per bank, so lookups never conflict).
template <int BITS, int B>
__global__ void __launch_bounds__(256)
    gemv_rowwarp_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ lut,
                        const int32_t* __restrict__ rowptr, const int32_t* __restrict__ col,
                        const uint16_t* __restrict__ val, int64_t nnz, const uint16_t* __restrict__ x,
                        int64_t ldx, uint16_t* __restrict__ y, int64_t ldy, int32_t n_out, int32_t k_in) {
    constexpr int L = 1 << BITS;
    __shared__ float s_lut[8][L];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wpr = (int64_t)k_in * BITS / 32;
    for (int64_t row = (int64_t)blockIdx.x * 8 + warp; row < n_out; row += (int64_t)gridDim.x * 8) {
        __syncwarp();
        if (lane < L) s_lut[warp][lane] = h2f(lut[row * L + lane]);
        __syncwarp();
        float acc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
        const uint32_t* rw = codes + row * wpr;
        if constexpr (BITS == 4) {
            for (int64_t u = lane; u < wpr; u += 32) {
                const uint32_t w = ldg_u32(rw + u);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float wv = s_lut[warp][(w >> (4 * j)) & 15u];
                    const int64_t k = u * 8 + j;
#pragma unroll
                    for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, h2f(__ldg(x + b * ldx + k)), acc[b]);
                }
            }
        } else {
            const int64_t units = k_in / 32;
            for (int64_t u = lane; u < units; u += 32) {
                const uint32_t w0 = ldg_u32(rw + 3 * u), w1 = ldg_u32(rw + 3 * u + 1), w2 = ldg_u32(rw + 3 * u + 2);
                Unroll3<0, 3>::run(w0, w1, w2, [&](int j, uint32_t c) {
                    const float wv = s_lut[warp][c];
                    const int64_t k = u * 32 + j;
#pragma unroll
                    for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, h2f(__ldg(x + b * ldx + k)), acc[b]);
                });
            }
        }
        if (nnz > 0) {
            const int32_t j0 = rowptr[row], j1 = rowptr[row + 1];
            for (int32_t j = j0 + lane; j < j1; j += 32) {
                const float v = h2f(val[j]);
                const int32_t c = col[j];
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] = fmaf(v, h2f(__ldg(x + b * ldx + c)), acc[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const float s = warp_sum(acc[b]);
            if (lane == 0) y[b * ldy + row] = f2h_rn(s);
        }
    }
}

// ------------------------------------------------------ fp16 dense yardstick
// y = W x with W fp16 [n_out][ldw]; one warp per row, 16-byte weight loads
// when the row is 16-byte aligned, fp32 accumulation.
template <int B>
__global__ void __launch_bounds__(256)
    fp16_gemv_kernel(const uint16_t* __restrict__ w, int64_t ldw, const uint16_t* __restrict__ x, int64_t ldx,
                     uint16_t* __restrict__ y, int64_t ldy, int32_t n_out, int32_t k_in, int vec_ok) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t row = (int64_t)blockIdx.x * 8 + warp; row < n_out; row += (int64_t)gridDim.x * 8) {
        const uint16_t* wr = w + row * ldw;
        float acc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
        int64_t k0 = 0;
        if (vec_ok) {
            const int64_t nvec = k_in / 8;
            for (int64_t v = lane; v < nvec; v += 32) {
                const uint4 q = ldg_stream_u128(wr + v * 8);
                const uint32_t qs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    const uint4 xq = ldg_u128(x + b * ldx + v * 8);
                    const uint32_t xs[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 wf = __half22float2(*reinterpret_cast<const __half2*>(&qs[e]));
                        const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&xs[e]));
                        acc[b] = fmaf(wf.x, xf.x, acc[b]);
                        acc[b] = fmaf(wf.y, xf.y, acc[b]);
                    }
                }
            }
            k0 = nvec * 8;
        }
        for (int64_t k = k0 + lane; k < k_in; k += 32) {
            const float wv = h2f(wr[k]);
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = fmaf(wv, h2f(__ldg(x + b * ldx + k)), acc[b]);
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const float s = warp_sum(acc[b]);
            if (lane == 0) y[b * ldy + row] = f2h_rn(s);
        }
    }
}

}  // namespace sqz
