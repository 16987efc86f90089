// kernels_tc.cuh -- the fused Dense-and-Sparse GEMV for sm_100a.
//
// y = (Q + S) x ("SqueezeLLM: Dense-and-Sparse Quantization", summary page,
// §3.4 "Kernel Implementation": LUT-based dense kernel, balanced sparse
// kernel, both fused into one launch).
//
// Work decomposition
//   * Rows are grouped in tiles of 16 (the M of an m16n8k16 MMA); columns in
//     super-groups of 256 (16 k16-steps).  A unit = (tile, super-group).
//   * Units are numbered tile-major and split into equal contiguous ranges:
//     one range per CTA (one CTA per SM), then one sub-range per warp.
//     Every SM and every warp streams the same number of code bytes.
//   * A tile whose units fall in several warps or CTAs is combined
//     deterministically: warps through shared memory, CTAs through a small
//     global partial buffer where the last CTA to arrive (atomic counter,
//     reset by that CTA) adds the parts in CTA order.  No thread ever waits
//     for another CTA.
//
// Streaming: each warp owns a ring of shared-memory stages filled by
// cp.async.bulk (TMA, 1-D) copies that complete on per-stage mbarriers; all
// waits are bounded and record a status bit instead of hanging.
//
// Decode (kernel-native code layout, built by repack_codes_kernel): for each
// k16-step a lane holds 4 codes of row g and 4 of row g+8 (g = lane/4) at
// columns 4*t4..4*t4+3 (t4 = lane%4) of the step.  A code indexes the row's
// LUT kept in registers as byte planes (low bytes, high bytes); `prmt`
// gathers the bytes of four weights at once and a second `prmt` interleaves
// them into fp16 pairs, which are exactly the A fragment of the MMA once
// the MMA's k order is permuted to match (the same permutation is applied
// to x, so the product is unchanged).
//
// MAC: fp16 x fp16 products are exact in fp32; accumulation is fp32, either
// on the tensor cores (mma.sync m16n8k16, batch columns in N) or on the CUDA
// cores (mixed-precision fma.rn.f32.f16, batch 1 only).
//
// Sparse part: the CSR entries of the rows whose tiles start in a CTA are
// split evenly over the CTA's threads (a fixed number of nonzeros per
// thread, independent of how skewed the rows are).  Each thread sums its
// entries per row; rows cut at thread boundaries are combined in thread
// order -- the balanced scheme of the pages, made deterministic.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace sqz {
namespace tc {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kCsrThreads = 256;  // threads that share the sparse part
constexpr int kTileRows = 16;
constexpr int kSgSteps = 16;   // k16-steps per super-group
constexpr int kSgCols = 256;   // columns per super-group
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kMaxGrid = 256;  // CTAs (one per SM)
constexpr int kCsrCap = 4096;  // CSR entries per CTA staged in shared memory

constexpr int kStatusWaitTimeout = 1;

template <int BITS>
struct Fmt;
template <>
struct Fmt<3> {
    static constexpr int kVecs = 3;        // uint4 per lane per super-group
    static constexpr int kSgBytes = 1536;  // 16 rows x 256 cols x 3 bits
    static constexpr int kLutBytes = 16;   // per row: 8 low bytes, 8 high bytes
};
template <>
struct Fmt<4> {
    static constexpr int kVecs = 4;
    static constexpr int kSgBytes = 2048;
    static constexpr int kLutBytes = 32;   // 16 low bytes, 16 high bytes
};

// ------------------------------------------------------------ shared plan
// Sizes that the host (for the launch) and the kernel (to carve shared
// memory) must agree on.
struct Plan {
    int64_t units;      // ntiles * nsg
    int grid;           // CTAs
    int stages;         // ring stages per warp
    int ctiles_max;     // max tiles touched by one CTA
    int x_stride;       // shared-memory row stride of x, in halves
    int bmax;           // 8 * NT
    // byte offsets
    int off_ring, off_x, off_lut, off_rp, off_col, off_val, off_head, off_tail, off_headrow, off_tailrow, off_rowsum, off_ctile,
        off_slots, off_flag, total;
};

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

__host__ __device__ inline Plan make_plan(int bits, int n_out, int k_in, int batch, int nt, int sms, int stages) {
    Plan P{};
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int nsteps = k_in / 16;
    const int nsg = (nsteps + kSgSteps - 1) / kSgSteps;
    const int sg_bytes = bits == 3 ? 1536 : 2048;
    const int lut_bytes = bits == 3 ? 16 : 32;
    P.units = (int64_t)ntiles * nsg;
    P.grid = (int)(P.units < sms ? P.units : sms);
    if (P.grid < 1) P.grid = 1;
    P.stages = stages;
    const int64_t upc = (P.units + P.grid - 1) / P.grid;
    P.ctiles_max = nsg > 0 ? (int)((upc + nsg - 1) / nsg) + 1 : 1;
    P.bmax = 8 * nt;
    // x rows: stride = 32 (mod 128) bytes keeps the batch rows of one
    // fragment load in different banks.
    int xs_bytes = round_up(k_in * 2, 128) + 32;
    P.x_stride = xs_bytes / 2;
    int off = 512;  // mbarriers: kWarps*stages + 1 (at most 65 * 8 B)
    P.off_ring = off;
    off += kWarps * stages * sg_bytes;
    P.off_x = off;
    off += round_up(batch * xs_bytes, 128);
    P.off_lut = off;
    off += round_up(P.ctiles_max * kTileRows * lut_bytes, 128);
    const int csr_rows = P.ctiles_max * kTileRows;
    P.off_rp = off;
    off += round_up((csr_rows + 8) * 4, 128);
    P.off_col = off;
    off += (kCsrCap + 8) * 4;
    P.off_val = off;
    off += (kCsrCap + 16) * 2;  // a slice starts up to 7 entries early and is rounded up to 8
    P.off_head = off;
    off += kCsrThreads * P.bmax * 4;
    P.off_tail = off;
    off += kCsrThreads * P.bmax * 4;
    P.off_headrow = off;
    off += kCsrThreads * 4;
    P.off_tailrow = off;
    off += kCsrThreads * 4;
    P.off_rowsum = off;
    off += round_up(csr_rows * P.bmax * 4, 128);
    P.off_ctile = off;
    off += P.ctiles_max * kTileRows * P.bmax * 4;
    P.off_slots = off;
    off += kWarps * 2 * kTileRows * P.bmax * 4;
    P.off_flag = off;
    off += 128;
    P.total = off;
    return P;
}

struct Params {
    const uint8_t* codes;    // [ntiles][nsg][sg_bytes], kernel-native layout
    const uint8_t* lutp;     // [ntiles*16][lut_bytes], byte planes
    const int32_t* rowptr;   // canonical CSR (device copies owned by the layer)
    const int32_t* col;
    const uint16_t* val;
    int64_t nnz;
    const uint16_t* x;
    int64_t ldx;
    uint16_t* y;
    int64_t ldy;
    float* part;             // [grid][2][16][16] cross-CTA partial sums
    int* tile_cnt;           // [ntiles] arrival counters, zero between calls
    int* status;             // error bits (bounded waits that gave up)
    int n_out, k_in, nsteps, nsg, ntiles, batch;
    int x_bulk;              // 1: every x row is 16-byte aligned -> bulk copies
    Plan plan;
    // rowptr at the first row owned by each CTA (the rows of the tiles whose
    // first unit is in the CTA), and at n_out for c = grid: the CTA's CSR
    // entries are [csr_rp[c], csr_rp[c+1]).  Computed once per layer.
    int csr_rp[kMaxGrid + 1];
};

// ------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false if the phase did not complete within kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
    return d;
}

// ----------------------------------------------------------------- decode
// Row LUT as byte planes.  Tab3: l0 = low bytes of entries 0..3, l1 = 4..7,
// h0/h1 the high bytes.  Tab4: l0..l3 low bytes of entries 0..15, h0..h3.
struct Tab3 {
    uint32_t l0, l1, h0, h1;
};
struct Tab4 {
    uint32_t l0, l1, l2, l3, h0, h1, h2, h3;
};

__device__ __forceinline__ Tab3 load_tab3(const uint8_t* row) {
    const uint4 v = *reinterpret_cast<const uint4*>(row);
    return Tab3{v.x, v.y, v.z, v.w};
}
__device__ __forceinline__ Tab4 load_tab4(const uint8_t* row) {
    const uint4 a = *reinterpret_cast<const uint4*>(row);
    const uint4 b = *reinterpret_cast<const uint4*>(row + 16);
    return Tab4{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
}

// Four 3-bit codes in the nibbles of sel (bit 3 of each nibble clear) ->
// fp16 pairs (w0,w1) and (w2,w3).
__device__ __forceinline__ void dec3(const Tab3& t, uint32_t sel, uint32_t& w01, uint32_t& w23) {
    const uint32_t lo = prmt(t.l0, t.l1, sel);
    const uint32_t hi = prmt(t.h0, t.h1, sel);
    w01 = prmt(lo, hi, 0x5140);
    w23 = prmt(lo, hi, 0x7362);
}

// Four 4-bit codes: s7 = codes with bit 3 cleared, pick = 0x3210 with bit 2
// of nibble i set when code i >= 8 (selects the upper half of the table).
__device__ __forceinline__ void dec4(const Tab4& t, uint32_t s7, uint32_t pick, uint32_t& w01, uint32_t& w23) {
    const uint32_t lo = prmt(prmt(t.l0, t.l1, s7), prmt(t.l2, t.l3, s7), pick);
    const uint32_t hi = prmt(prmt(t.h0, t.h1, s7), prmt(t.h2, t.h3, s7), pick);
    w01 = prmt(lo, hi, 0x5140);
    w23 = prmt(lo, hi, 0x7362);
}

// Selectors of one 3-bit quad (steps 4q..4q+3) from the lane's 3 words:
// step j<3 uses bits 0..2 of the nibbles of word j; step 3's codes are
// spread over bit 3 of the nibbles of the three words (bit j of the code
// in word j).  Low 16 bits: row g; high 16 bits: row g+8.
__device__ __forceinline__ uint32_t sel3_extra(uint32_t w0, uint32_t w1, uint32_t w2) {
    return ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
}

// Decode one k16-step of a lane: a0/a2 = row g pairs, a1/a3 = row g+8 pairs.
template <int BITS, class TAB>
__device__ __forceinline__ void decode_step(const TAB& tg, const TAB& tg8, uint32_t word, uint32_t& a0, uint32_t& a1,
                                            uint32_t& a2, uint32_t& a3) {
    if constexpr (BITS == 3) {
        dec3(tg, word & 0x7777u, a0, a2);
        dec3(tg8, (word >> 16) & 0x7777u, a1, a3);
    } else {
        dec4(tg, word & 0x7777u, 0x3210u | ((word >> 1) & 0x4444u), a0, a2);
        dec4(tg8, (word >> 16) & 0x7777u, 0x3210u | ((word >> 17) & 0x4444u), a1, a3);
    }
}

// Step word j (0..15) of a super-group for a lane, from its uint4 vectors.
// 3-bit: word 4q+j' (j' < 3) is stored; word 4q+3 is rebuilt from the three.
template <int BITS>
__device__ __forceinline__ uint32_t step_word(const uint32_t* w, int step) {
    if constexpr (BITS == 4) {
        return w[step];
    } else {
        const int q = step >> 2, j = step & 3;
        if (j < 3) return w[3 * q + j];
        return sel3_extra(w[3 * q], w[3 * q + 1], w[3 * q + 2]);
    }
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc += w.lo * x.lo + w.hi * x.hi with fp16 operands and an fp32
// accumulator (products exact), on the CUDA cores.
__device__ __forceinline__ void fma2_mixed(float& acc, uint32_t w, uint32_t x) {
    asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
        " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %0, wh, xh, %0;\n}"
        : "+f"(acc)
        : "r"(w), "r"(x));
}

// ------------------------------------------------------------ repacking
// Code (row, k) of the canonical LSB-first bitstream layout.
template <int BITS>
__device__ __forceinline__ uint32_t canon_code(const uint32_t* codes, int64_t wpr, int row, int k) {
    const int64_t bit = (int64_t)k * BITS;
    const uint32_t* rw = codes + (int64_t)row * wpr;
    const int64_t wi = bit >> 5;
    const int sh = (int)(bit & 31);
    uint32_t v = rw[wi] >> sh;
    if (sh + BITS > 32) v |= rw[wi + 1] << (32 - sh);
    return v & ((1u << BITS) - 1u);
}

// One thread per output word of the kernel-native layout.
template <int BITS>
__global__ void repack_codes_kernel(const uint32_t* __restrict__ canon, int32_t n_out, int32_t k_in, int nsg,
                                    int64_t total_words, uint32_t* __restrict__ out) {
    using F = Fmt<BITS>;
    const int64_t wpr = (int64_t)k_in * BITS / 32;
    const int nsteps = k_in / 16;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < total_words;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t unit = wi / (F::kVecs * 128);
        const int rem = (int)(wi % (F::kVecs * 128));
        const int m = rem >> 7, lane = (rem >> 2) & 31, e = rem & 3;
        const int lw = 4 * m + e;  // word index within the lane's list
        const int tile = (int)(unit / nsg), sg = (int)(unit % nsg);
        const int g = lane >> 2, t4 = lane & 3;
        auto code_or0 = [&](int n, int step) -> uint32_t {
            const int row = tile * kTileRows + g + 8 * (n >> 2);
            const int gstep = sg * kSgSteps + step;
            if (row >= n_out || gstep >= nsteps) return 0u;
            return canon_code<BITS>(canon, wpr, row, gstep * 16 + 4 * t4 + (n & 3));
        };
        uint32_t word = 0;
        if constexpr (BITS == 4) {
            for (int n = 0; n < 8; ++n) word |= code_or0(n, lw) << (4 * n);
        } else {
            const int q = lw / 3, j = lw % 3;
            for (int n = 0; n < 8; ++n) {
                const uint32_t c = code_or0(n, 4 * q + j);
                const uint32_t x = (code_or0(n, 4 * q + 3) >> j) & 1u;
                word |= (c | (x << 3)) << (4 * n);
            }
        }
        out[wi] = word;
    }
}

// LUT rows -> byte planes; rows beyond n_out (tile padding) are zero.
template <int BITS>
__global__ void repack_lut_kernel(const uint16_t* __restrict__ lut, int32_t n_out, int32_t rows_padded,
                                  uint8_t* __restrict__ out) {
    constexpr int L = 1 << BITS;
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows_padded; r += gridDim.x * blockDim.x) {
        uint8_t* o = out + (int64_t)r * 2 * L;
        for (int e = 0; e < L; ++e) {
            const uint16_t v = r < n_out ? lut[(int64_t)r * L + e] : (uint16_t)0;
            o[e] = (uint8_t)(v & 0xff);
            o[L + e] = (uint8_t)(v >> 8);
        }
    }
}

// Dequantized weights from the kernel-native layout, with the GEMV's own
// decoder: w_out[row][k] = lut[row][code(row,k)].
template <int BITS>
__global__ void dequant_native_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ lutp,
                                      int32_t n_out, int32_t k_in, int nsg, int64_t units,
                                      uint16_t* __restrict__ w_out) {
    using F = Fmt<BITS>;
    using TAB = typename std::conditional<BITS == 3, Tab3, Tab4>::type;
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int nsteps = k_in / 16;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t u = warp0; u < units; u += nwarps) {
        const int tile = (int)(u / nsg), sg = (int)(u % nsg);
        uint32_t w[4 * F::kVecs];
        const uint8_t* base = codes + u * F::kSgBytes + lane * 16;
        for (int m = 0; m < F::kVecs; ++m) {
            const uint4 v = *reinterpret_cast<const uint4*>(base + m * 512);
            w[4 * m] = v.x, w[4 * m + 1] = v.y, w[4 * m + 2] = v.z, w[4 * m + 3] = v.w;
        }
        const int rg = tile * kTileRows + g, rg8 = rg + 8;
        TAB tg, tg8;
        if constexpr (BITS == 3) {
            tg = load_tab3(lutp + (int64_t)rg * F::kLutBytes);
            tg8 = load_tab3(lutp + (int64_t)rg8 * F::kLutBytes);
        } else {
            tg = load_tab4(lutp + (int64_t)rg * F::kLutBytes);
            tg8 = load_tab4(lutp + (int64_t)rg8 * F::kLutBytes);
        }
#pragma unroll
        for (int st = 0; st < kSgSteps; ++st) {
            const int gstep = sg * kSgSteps + st;
            if (gstep >= nsteps) break;
            uint32_t a0, a1, a2, a3;
            decode_step<BITS>(tg, tg8, step_word<BITS>(w, st), a0, a1, a2, a3);
            const int k = gstep * 16 + 4 * t4;
            if (rg < n_out) {
                uint32_t* o = reinterpret_cast<uint32_t*>(w_out + (int64_t)rg * k_in + k);
                o[0] = a0, o[1] = a2;
            }
            if (rg8 < n_out) {
                uint32_t* o = reinterpret_cast<uint32_t*>(w_out + (int64_t)rg8 * k_in + k);
                o[0] = a1, o[1] = a3;
            }
        }
    }
}

// ------------------------------------------------------------ main kernel
__device__ __forceinline__ int cta_begin(int units, int grid, int c) { return (int)((int64_t)units * c / grid); }

// CTA whose unit range contains u.
__device__ __forceinline__ int cta_of(int units, int grid, int u) {
    int c = (int)(((int64_t)u * grid) / units);
    while (c + 1 < grid && cta_begin(units, grid, c + 1) <= u) ++c;
    while (c > 0 && cta_begin(units, grid, c) > u) --c;
    return c;
}

template <int BITS, int NT, bool TC>
__global__ void __launch_bounds__(kThreads, 1) gemv_fused_kernel(const __grid_constant__ Params p) {
    using F = Fmt<BITS>;
    using TAB = typename std::conditional<BITS == 3, Tab3, Tab4>::type;
    constexpr int BM = 8 * NT;             // batch columns per accumulator set
    constexpr int TE = kTileRows * BM;      // elements of one tile's result
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan& P = p.plan;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int G = gridDim.x, c = blockIdx.x;
    const int nsg = p.nsg;
    const int U = (int)P.units;
    const int u0 = cta_begin(U, G, c), u1 = cta_begin(U, G, c + 1);
    const int cn = u1 - u0;
    const int wu0 = u0 + cn * warp / kWarps, wu1 = u0 + cn * (warp + 1) / kWarps;
    const int t_first = u0 / nsg, t_last = (u1 - 1) / nsg;
    const int ctiles = t_last - t_first + 1;
    const int stages = P.stages;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint64_t* wbar = bars + warp * stages;
    uint64_t* xbar = bars + kWarps * stages;
    uint8_t* ring = smem + P.off_ring + warp * stages * F::kSgBytes;
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.off_x);
    uint8_t* luts = smem + P.off_lut;
    float* s_head = reinterpret_cast<float*>(smem + P.off_head);
    float* s_tail = reinterpret_cast<float*>(smem + P.off_tail);
    int* s_headrow = reinterpret_cast<int*>(smem + P.off_headrow);
    int* s_tailrow = reinterpret_cast<int*>(smem + P.off_tailrow);
    float* s_rowsum = reinterpret_cast<float*>(smem + P.off_rowsum);
    float* s_ctile = reinterpret_cast<float*>(smem + P.off_ctile);
    float* s_slots = reinterpret_cast<float*>(smem + P.off_slots);
    int* s_flag = reinterpret_cast<int*>(smem + P.off_flag);

    // ---- barriers
    if (lane == 0)
        for (int s = 0; s < stages; ++s) mbar_init(&wbar[s], 1);
    if (tid == 0) mbar_init(xbar, 1);
    fence_mbar_init();
    __syncthreads();

    // ---- sparse rows owned by this CTA: those of the tiles whose first unit
    // lies in [u0, u1); their CSR entries are [csr_rp[c], csr_rp[c+1]).
    const int ta = (u0 + nsg - 1) / nsg, tb = t_last;
    const int ra = min(p.n_out, ta * kTileRows);
    const int nrows = ta <= tb ? min(p.n_out, (tb + 1) * kTileRows) - ra : 0;
    const int p0 = p.csr_rp[c], p1 = p.csr_rp[c + 1];
    const int nz = p1 - p0;
    const bool has_csr = p.nnz > 0 && nrows > 0;
    const bool csr_smem = has_csr && nz <= kCsrCap;
    // staged slices start at 16-byte aligned source addresses; these are the
    // element offsets of the first wanted entry inside the staged buffers
    const int rp_off = ra & 3, col_off = p0 & 3, val_off = p0 & 7;

    // ---- CTA-wide copies: LUT planes of the CTA's tiles, x (when every row
    // is 16-byte aligned) and the CTA's CSR slices
    const uint32_t lut_bytes = (uint32_t)ctiles * kTileRows * F::kLutBytes;
    if (tid == 0) {
        uint32_t tx = lut_bytes + (p.x_bulk ? (uint32_t)p.batch * p.k_in * 2 : 0u);
        const uint32_t rp_bytes = has_csr ? (uint32_t)round_up(nrows + 1 + rp_off, 4) * 4 : 0u;
        const uint32_t col_bytes = csr_smem ? (uint32_t)round_up(nz + col_off, 4) * 4 : 0u;
        const uint32_t val_bytes = csr_smem ? (uint32_t)round_up(nz + val_off, 8) * 2 : 0u;
        tx += rp_bytes + col_bytes + val_bytes;
        mbar_expect_tx(xbar, tx);
        bulk_g2s(luts, p.lutp + (int64_t)t_first * kTileRows * F::kLutBytes, lut_bytes, xbar);
        if (p.x_bulk)
            for (int b = 0; b < p.batch; ++b) bulk_g2s(xs + b * P.x_stride, p.x + b * p.ldx, p.k_in * 2, xbar);
        if (rp_bytes) bulk_g2s(smem + P.off_rp, p.rowptr + (ra - rp_off), rp_bytes, xbar);
        if (col_bytes) bulk_g2s(smem + P.off_col, p.col + (p0 - col_off), col_bytes, xbar);
        if (val_bytes) bulk_g2s(smem + P.off_val, p.val + (p0 - val_off), val_bytes, xbar);
    }
    // ---- per-warp ring prologue
    const int nwu = wu1 - wu0;
    int issued = nwu < stages ? nwu : stages;
    if (lane == 0)
        for (int s = 0; s < issued; ++s) {
            mbar_expect_tx(&wbar[s], F::kSgBytes);
            bulk_g2s(ring + s * F::kSgBytes, p.codes + (int64_t)(wu0 + s) * F::kSgBytes, F::kSgBytes, &wbar[s]);
        }
    if (!p.x_bulk) {
        for (int i = tid; i < p.batch * p.k_in; i += kThreads) {
            const int b = i / p.k_in, k = i - b * p.k_in;
            xs[b * P.x_stride + k] = p.x[b * p.ldx + k];
        }
    }
    if (has_csr) {
        for (int i = tid; i < nrows * BM; i += kThreads) s_rowsum[i] = 0.f;
        if (tid < kCsrThreads) {
            s_headrow[tid] = -1;
            s_tailrow[tid] = -1;
        }
    }
    const bool ok = __syncthreads_and(mbar_wait(xbar, 0) ? 1 : 0) != 0;
    if (!ok && tid == 0) atomicOr(p.status, kStatusWaitTimeout);

    // ---- sparse part: a fixed share of nonzeros per thread (balanced)
    const int B = p.batch;
    const int* s_rp = reinterpret_cast<const int*>(smem + P.off_rp) + rp_off;
    const int* csr_col = csr_smem ? reinterpret_cast<const int*>(smem + P.off_col) + col_off - p0 : p.col;
    const uint16_t* csr_val =
        csr_smem ? reinterpret_cast<const uint16_t*>(smem + P.off_val) + val_off - p0 : p.val;
    const int e_per = has_csr ? max(1, (nz + kCsrThreads - 1) / kCsrThreads) : 1;
    if (has_csr && ok && tid < kCsrThreads) {
        const int a = p0 + tid * e_per;
        const int b_end = min(p1, a + e_per);
        if (a < b_end) {
            // row (relative to ra) containing entry a: largest r with s_rp[r] <= a
            int lo = 0, hi = nrows - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_rp[mid] <= a) lo = mid; else hi = mid - 1;
            }
            int cur = lo;
            bool first = true;
            float acc[BM];
#pragma unroll
            for (int b = 0; b < BM; ++b) acc[b] = 0.f;
            auto emit = [&](bool last) {
                if (first) {
                    s_headrow[tid] = cur;
#pragma unroll
                    for (int b = 0; b < BM; ++b) s_head[tid * BM + b] = acc[b];
                } else if (last) {
                    s_tailrow[tid] = cur;
#pragma unroll
                    for (int b = 0; b < BM; ++b) s_tail[tid * BM + b] = acc[b];
                } else {
#pragma unroll
                    for (int b = 0; b < BM; ++b) s_rowsum[cur * BM + b] = acc[b];
                }
            };
            for (int base = a; base < b_end; base += 8) {
                int cc[8];
                float vv[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int q = base + j;
                    cc[j] = q < b_end ? csr_col[q] : 0;
                    vv[j] = q < b_end ? h2f(csr_val[q]) : 0.f;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int q = base + j;
                    if (q >= b_end) break;
                    while (q >= s_rp[cur + 1]) {
                        emit(false);
                        first = false;
#pragma unroll
                        for (int b = 0; b < BM; ++b) acc[b] = 0.f;
                        ++cur;
                    }
#pragma unroll
                    for (int b = 0; b < BM; ++b)
                        if (b < B) acc[b] = fmaf(vv[j], h2f(xs[b * P.x_stride + cc[j]]), acc[b]);
                }
            }
            emit(true);
        }
    }

    // ---- dense part
    const int xrow = (g < B) ? g : 0;  // batch column of this lane's B fragment (n = g)
    const int xrow2 = (NT == 2 && g + 8 < B) ? g + 8 : 0;
    const bool xon = g < B, xon2 = (NT == 2) && (g + 8 < B);
    const int wfirst = nwu > 0 ? wu0 / nsg : -1;
    int tile = wfirst, sg = nwu > 0 ? wu0 - wfirst * nsg : 0;
    int s = 0, consumed = 0;
    uint32_t par = 0;
    bool alive = ok;
    int fail_at = -1;
    for (int u = wu0; u < wu1;) {
        const int run = min(wu1 - u, nsg - sg);  // units of `tile` in this warp's range
        const uint8_t* lt = luts + (tile - t_first) * kTileRows * F::kLutBytes;
        TAB tg, tg8;
        if constexpr (BITS == 3) {
            tg = load_tab3(lt + g * F::kLutBytes);
            tg8 = load_tab3(lt + (g + 8) * F::kLutBytes);
        } else {
            tg = load_tab4(lt + g * F::kLutBytes);
            tg8 = load_tab4(lt + (g + 8) * F::kLutBytes);
        }
        float d0[NT][4], d1[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) d0[n][i] = d1[n][i] = 0.f;
        float f0 = 0.f, f1 = 0.f;  // CUDA-core accumulators (rows g, g+8)

        for (int r = 0; r < run; ++r, ++sg, ++consumed) {
            if (alive) {
                const bool got = __all_sync(0xffffffffu, mbar_wait(&wbar[s], par));
                if (!got) {
                    alive = false;
                    fail_at = consumed;
                    if (lane == 0) atomicOr(p.status, kStatusWaitTimeout);
                }
            }
            uint32_t w[4 * F::kVecs];
            const uint8_t* sb = ring + s * F::kSgBytes + lane * 16;
#pragma unroll
            for (int m = 0; m < F::kVecs; ++m) {
                const uint4 v = *reinterpret_cast<const uint4*>(sb + m * 512);
                w[4 * m] = v.x, w[4 * m + 1] = v.y, w[4 * m + 2] = v.z, w[4 * m + 3] = v.w;
            }
            __syncwarp();
            if (alive && issued < nwu) {
                if (lane == 0) {
                    fence_proxy_async();
                    mbar_expect_tx(&wbar[s], F::kSgBytes);
                    bulk_g2s(ring + s * F::kSgBytes, p.codes + (int64_t)(wu0 + issued) * F::kSgBytes, F::kSgBytes,
                             &wbar[s]);
                }
                ++issued;
            }
            if (++s == stages) {
                s = 0;
                par ^= 1u;
            }
            const int step0 = sg * kSgSteps;
            const int nvalid = min(kSgSteps, p.nsteps - step0);
            const uint16_t* xb0 = xs + xrow * P.x_stride + step0 * 16 + 4 * t4;
            const uint16_t* xb1 = xs + xrow2 * P.x_stride + step0 * 16 + 4 * t4;
#pragma unroll
            for (int st = 0; st < kSgSteps; ++st) {
                if (st >= nvalid) break;  // ragged last super-group only
                uint32_t a0, a1, a2, a3;
                decode_step<BITS>(tg, tg8, step_word<BITS>(w, st), a0, a1, a2, a3);
                if constexpr (TC) {
                    const uint2 xv = xon ? *reinterpret_cast<const uint2*>(xb0 + st * 16) : make_uint2(0u, 0u);
                    if (st & 1)
                        mma16816(d1[0], a0, a1, a2, a3, xv.x, xv.y);
                    else
                        mma16816(d0[0], a0, a1, a2, a3, xv.x, xv.y);
                    if constexpr (NT == 2) {
                        const uint2 xw = xon2 ? *reinterpret_cast<const uint2*>(xb1 + st * 16) : make_uint2(0u, 0u);
                        if (st & 1)
                            mma16816(d1[1], a0, a1, a2, a3, xw.x, xw.y);
                        else
                            mma16816(d0[1], a0, a1, a2, a3, xw.x, xw.y);
                    }
                } else {
                    const uint2 xv = *reinterpret_cast<const uint2*>(xs + step0 * 16 + 4 * t4 + st * 16);
                    fma2_mixed(f0, a0, xv.x);
                    fma2_mixed(f0, a2, xv.y);
                    fma2_mixed(f1, a1, xv.x);
                    fma2_mixed(f1, a3, xv.y);
                }
            }
        }
        // ---- this warp's contribution to `tile`
        float rr[NT][4];
        if constexpr (TC) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) rr[n][i] = d0[n][i] + d1[n][i];
        } else {
            f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
            f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
            rr[0][0] = t4 == 0 ? f0 : 0.f;
            rr[0][1] = 0.f;
            rr[0][2] = t4 == 0 ? f1 : 0.f;
            rr[0][3] = 0.f;
        }
        // exclusive: this warp holds all of the CTA's units of the tile
        const bool excl = u == max(u0, tile * nsg) && u + run == min(u1, (tile + 1) * nsg);
        float* dst = excl ? s_ctile + (tile - t_first) * TE
                          : s_slots + (warp * 2 + (tile == wfirst ? 0 : 1)) * TE;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int col = 8 * n + 2 * t4;
            dst[g * BM + col] = rr[n][0];
            dst[g * BM + col + 1] = rr[n][1];
            dst[(g + 8) * BM + col] = rr[n][2];
            dst[(g + 8) * BM + col + 1] = rr[n][3];
        }
        u += run;
        ++tile;
        sg = 0;
    }
    // A wait that gave up leaves copies in flight into this warp's ring (and
    // possibly the CTA-wide ones): wait for them, again with a bound, before
    // the shared memory can be retired.
    if (!alive && fail_at >= 0)
        for (int j = fail_at; j < issued; ++j) (void)mbar_wait(&wbar[j % stages], (uint32_t)(j / stages) & 1u);
    if (!ok) (void)mbar_wait(xbar, 0);
    __syncthreads();

    // ---- sparse rows cut at thread boundaries: combine in thread order
    if (has_csr) {
        for (int i = tid; i < nrows; i += kThreads) {
            const int rs = s_rp[i], re = s_rp[i + 1];
            if (re > rs) {
                const int tau_a = (rs - p0) / e_per, tau_b = min(kCsrThreads - 1, (re - 1 - p0) / e_per);
                for (int tau = tau_a; tau <= tau_b; ++tau) {
                    if (s_headrow[tau] == i)
#pragma unroll
                        for (int b = 0; b < BM; ++b) s_rowsum[i * BM + b] += s_head[tau * BM + b];
                    if (s_tailrow[tau] == i)
#pragma unroll
                        for (int b = 0; b < BM; ++b) s_rowsum[i * BM + b] += s_tail[tau * BM + b];
                }
            }
        }
        __syncthreads();
    }

    // ---- per tile: sum the warps' parts (warp order), add the sparse rows,
    // then write y (tile complete in this CTA) or publish the partial
    for (int tl = 0; tl < ctiles; ++tl) {
        const int tile_i = t_first + tl;
        const int ta_u = max(u0, tile_i * nsg), tb_u = min(u1, (tile_i + 1) * nsg);
        const bool whole = ta_u == tile_i * nsg && tb_u == (tile_i + 1) * nsg;
        for (int e = tid; e < TE; e += kThreads) {
            const int row_l = e / BM, col = e - row_l * BM;
            float sum = 0.f;
            bool direct = false;
            for (int wv = 0; wv < kWarps; ++wv) {
                const int a = u0 + cn * wv / kWarps, b = u0 + cn * (wv + 1) / kWarps;
                const int lo = max(a, ta_u), hi = min(b, tb_u);
                if (lo >= hi) continue;
                if (lo == ta_u && hi == tb_u) {
                    direct = true;
                    break;
                }
                const int wf = a / nsg;
                sum += s_slots[(wv * 2 + (tile_i == wf ? 0 : 1)) * TE + e];
            }
            if (direct) sum = s_ctile[tl * TE + e];
            const int row = tile_i * kTileRows + row_l;
            if (has_csr && row >= ra && row < ra + nrows) sum += s_rowsum[(row - ra) * BM + col];
            if (whole) {
                if (row < p.n_out && col < B) p.y[col * p.ldy + row] = f2h_rn(sum);
            } else {
                const int slot = (tile_i == t_first) ? 0 : 1;
                p.part[(((int64_t)c * 2 + slot) * kTileRows + row_l) * 16 + col] = sum;
            }
        }
    }
    // ---- tiles shared with other CTAs: the last CTA to arrive adds the parts
    for (int side = 0; side < 2; ++side) {
        const int tile_i = side == 0 ? t_first : t_last;
        if (side == 1 && t_last == t_first) break;
        const bool whole = u0 <= tile_i * nsg && (tile_i + 1) * nsg <= u1;
        if (whole) continue;
        __syncthreads();  // this CTA's partial is written
        if (tid == 0) {
            const int cf = cta_of(U, G, tile_i * nsg), cl = cta_of(U, G, (tile_i + 1) * nsg - 1);
            __threadfence();  // release the CTA's partial before counting
            const int old = atomicAdd(&p.tile_cnt[tile_i], 1);
            const int last = old == cl - cf;
            if (last) __threadfence();  // acquire the other CTAs' partials
            *s_flag = last ? (cf | (cl << 16)) + 1 : 0;
        }
        __syncthreads();
        const int fl = *s_flag;
        if (fl) {
            const int cf = (fl - 1) & 0xffff, cl = (fl - 1) >> 16;
            for (int e = tid; e < TE; e += kThreads) {
                const int row_l = e / BM, col = e - row_l * BM;
                const int row = tile_i * kTileRows + row_l;
                float sum = 0.f;
                for (int cc = cf; cc <= cl; ++cc) {
                    const int slot = (tile_i == cta_begin(U, G, cc) / nsg) ? 0 : 1;
                    sum += __ldcg(p.part + (((int64_t)cc * 2 + slot) * kTileRows + row_l) * 16 + col);
                }
                if (row < p.n_out && col < B) p.y[col * p.ldy + row] = f2h_rn(sum);
            }
            if (tid == 0) p.tile_cnt[tile_i] = 0;
        }
    }
}

}  // namespace tc
}  // namespace sqz
