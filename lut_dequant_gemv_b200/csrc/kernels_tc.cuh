// kernels_tc.cuh -- the fused Dense-and-Sparse GEMV for sm_100a.
//
// y = (Q + S) x ("SqueezeLLM: Dense-and-Sparse Quantization", summary page,
// §3.4 "Kernel Implementation": LUT-based dense kernel, balanced sparse
// kernel, both fused into one launch).
//
// Work decomposition
//   * Rows are grouped in tiles of 16 (the M of an m16n8k16 MMA); columns in
//     super-groups of 256 (16 k16-steps).  A unit = (tile, super-group).
//   * Each CTA owns a contiguous run of whole tiles (runs differ by at most
//     one tile; grid = min(tiles, 2 CTAs per SM)) and its warps split the
//     CTA's units into equal contiguous ranges.  A tile is therefore
//     finished inside one CTA: the warps' partial sums are added in warp
//     order in shared memory -- deterministic, no global atomics.
//     Consecutive calls overlap through programmatic dependent launch, so
//     SMs that finish early start the next call's loads.
//
// Streaming: the codes are read with coalesced 128-bit loads straight into
// registers.  Each warp issues the loads of its first units before waiting
// for the previous kernel in the stream (programmatic dependent launch:
// the weights never depend on it), then keeps a fixed number of units in
// flight while it decodes.  The LUT planes and the CTA's CSR slices are
// bulk-copied (TMA, 1-D) into shared memory, x after the wait; the waits
// on those copies are bounded and record a status bit instead of hanging.
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

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = 2;
constexpr int kCsrThreads = kThreads;  // threads that share the sparse part
constexpr int kTileRows = 16;
constexpr int kSgSteps = 16;   // k16-steps per super-group
constexpr int kSgCols = 256;   // columns per super-group
constexpr uint32_t kSuspendNs = 1000000u;  // 1 ms per poll
constexpr uint32_t kWaitLimit = 2000u;
constexpr int kCsrCap = 2048;  // CSR entries per CTA staged in shared memory

constexpr int kStatusWaitTimeout = 1;

template <int BITS>
struct Fmt;
template <>
struct Fmt<3> {
    static constexpr int kVecs = 3;        // uint4 per lane per super-group
    static constexpr int kSgBytes = 1536;  // 16 rows x 256 cols x 3 bits
    static constexpr int kLutBytes = 16;   // per row: 8 low bytes, 8 high bytes
    static constexpr int kDepth = 4;       // units a warp keeps in flight (registers)
};
template <>
struct Fmt<4> {
    static constexpr int kVecs = 4;
    static constexpr int kSgBytes = 2048;
    static constexpr int kLutBytes = 32;   // 16 low bytes, 16 high bytes
    static constexpr int kDepth = 3;
};

// ------------------------------------------------------------ shared plan
// Sizes that the host (for the launch) and the kernel (to carve shared
// memory) must agree on.
struct Plan {
    int64_t units;      // ntiles * nsg
    int grid;           // CTAs
    int ctiles_max;     // max tiles touched by one CTA
    int x_stride;       // shared-memory row stride of x, in halves
    int cm;             // batch columns carried by the sparse part and the combine (1 or 8*NT)
    // byte offsets
    int off_x, off_lut, off_rp, off_col, off_val, off_head, off_tail, off_headrow, off_tailrow, off_rowsum, off_ctile,
        off_slots, off_wrange, off_tinfo, total;
};

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// First tile of CTA c when `ntiles` tiles are split over `grid` CTAs.
__host__ __device__ inline int tile_begin(int ntiles, int grid, int c) { return (int)((int64_t)ntiles * c / grid); }

// `ctas`: CTAs the device keeps resident (kCtasPerSm per SM).
__host__ __device__ inline Plan make_plan(int bits, int n_out, int k_in, int batch, int nt, bool single, int ctas) {
    Plan P{};
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int nsteps = k_in / 16;
    const int nsg = (nsteps + kSgSteps - 1) / kSgSteps;
    const int lut_bytes = bits == 3 ? 16 : 32;
    P.units = (int64_t)ntiles * nsg;
    P.grid = ntiles < ctas ? ntiles : ctas;
    if (P.grid < 1) P.grid = 1;
    P.ctiles_max = (ntiles + P.grid - 1) / P.grid;
    P.cm = single ? 1 : 8 * nt;
    // x rows: stride = 32 (mod 128) bytes keeps the batch rows of one
    // fragment load in different banks.
    int xs_bytes = round_up(k_in * 2, 128) + 32;
    P.x_stride = xs_bytes / 2;
    int off = 128;  // three mbarriers, CSR bounds
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
    off += kCsrThreads * P.cm * 4;
    P.off_tail = off;
    off += kCsrThreads * P.cm * 4;
    P.off_headrow = off;
    off += kCsrThreads * 4;
    P.off_tailrow = off;
    off += kCsrThreads * 4;
    P.off_rowsum = off;
    off += round_up(csr_rows * P.cm * 4, 128);
    P.off_ctile = off;
    off += P.ctiles_max * kTileRows * P.cm * 4;
    P.off_slots = off;
    off += kWarps * 2 * kTileRows * P.cm * 4;
    P.off_wrange = off;
    off += kWarps * 3 * 4;
    P.off_tinfo = off;
    off += round_up(P.ctiles_max * 4, 16);
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
    int* status;             // error bits (bounded waits that gave up)
    int n_out, k_in, nsteps, nsg, ntiles, batch;
    int x_bulk;              // 1: every x row is 16-byte aligned -> bulk copies
    Plan plan;
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
// One bounded poll: the thread is suspended until the phase completes or
// kSuspendNs nanoseconds pass, whichever comes first (no busy spinning that
// would take issue slots from the warps doing the arithmetic).
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}
// Bounded wait: false if the phase did not complete within kWaitLimit polls
// (at most kWaitLimit * kSuspendNs, about two seconds).
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
// Programmatic dependent launch: let the next kernel of the stream start
// (its CTAs may begin on SMs this grid leaves), and wait until the previous
// kernel of the stream has finished and its writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_previous() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

// Decode one k16-step of a lane from its selector word(s): a0/a2 = row g
// pairs, a1/a3 = row g+8 pairs.  3-bit: `m` holds the codes of row g in its
// low 16 bits and of row g+8 in its high 16 bits, bit 3 of every nibble
// clear.  4-bit: the step word `w`; bit 3 of a nibble selects the upper
// half of the table.
__device__ __forceinline__ void decode3(const Tab3& tg, const Tab3& tg8, uint32_t m, uint32_t& a0, uint32_t& a1,
                                        uint32_t& a2, uint32_t& a3) {
    dec3(tg, m, a0, a2);
    dec3(tg8, m >> 16, a1, a3);
}
__device__ __forceinline__ void decode4(const Tab4& tg, const Tab4& tg8, uint32_t w, uint32_t& a0, uint32_t& a1,
                                        uint32_t& a2, uint32_t& a3) {
    const uint32_t m = w & 0x77777777u;
    const uint32_t pk = ((w >> 1) & 0x44444444u) | 0x32103210u;
    dec4(tg, m, pk, a0, a2);
    dec4(tg8, m >> 16, pk >> 16, a1, a3);
}

// Step `st` (0..15) of a lane's super-group words.  3-bit: word 4q+j (j < 3)
// is stored as such; step 4q+3 is rebuilt from bit 3 of the three words.
template <int BITS, class TAB>
__device__ __forceinline__ void decode_step(const TAB& tg, const TAB& tg8, const uint32_t* w, int st, uint32_t& a0,
                                            uint32_t& a1, uint32_t& a2, uint32_t& a3) {
    if constexpr (BITS == 3) {
        const int q = st >> 2, j = st & 3;
        const uint32_t m = j < 3 ? (w[3 * q + j] & 0x77777777u) : sel3_extra(w[3 * q], w[3 * q + 1], w[3 * q + 2]);
        decode3(tg, tg8, m, a0, a1, a2, a3);
    } else {
        decode4(tg, tg8, w[st], a0, a1, a2, a3);
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
            decode_step<BITS>(tg, tg8, w, st, a0, a1, a2, a3);
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
// SB: batch 1 (one column carried through the sparse part and the combine).
template <int BITS, int NT, bool TC, bool SB>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) gemv_fused_kernel(const __grid_constant__ Params p) {
    using F = Fmt<BITS>;
    using TAB = typename std::conditional<BITS == 3, Tab3, Tab4>::type;
    constexpr int BM = 8 * NT;              // batch columns of the MMA accumulators
    constexpr int CM = SB ? 1 : BM;         // batch columns carried after the dense loop
    constexpr int TE = kTileRows * CM;      // elements of one tile's result
    constexpr int D = F::kDepth;            // units in flight per warp
    static_assert(!SB || NT == 1, "single-batch variant uses one n-tile");
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan& P = p.plan;

    // The next kernel in the stream may start as soon as SMs free up.
    pdl_launch_dependents();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int G = gridDim.x, c = blockIdx.x;
    const int nsg = p.nsg;
    const int t_first = tile_begin(p.ntiles, G, c), t_end = tile_begin(p.ntiles, G, c + 1);
    const int ctiles = t_end - t_first;
    const int u0 = t_first * nsg, u1 = t_end * nsg;  // whole tiles
    const int cn = u1 - u0;
    const int wu0 = u0 + cn * warp / kWarps, wu1 = u0 + cn * (warp + 1) / kWarps;
    const int nwu = wu1 - wu0;
    const int wfirst = nwu > 0 ? wu0 / nsg : -1;

    // ---- code prefetch: the first D units of this warp, straight into
    // registers (coalesced: each 128-bit load of the warp reads 512
    // consecutive bytes); weights never depend on the previous kernel
    uint4 R[D][F::kVecs];
#pragma unroll
    for (int j = 0; j < D; ++j) {
        if (j < nwu) {
            const uint8_t* src = p.codes + (int64_t)(wu0 + j) * F::kSgBytes + lane * 16;
#pragma unroll
            for (int m = 0; m < F::kVecs; ++m) R[j][m] = ldg_stream_u128(src + m * 512);
        }
    }

    uint64_t* lbar = reinterpret_cast<uint64_t*>(smem);      // LUT planes
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem) + 1;  // CSR slices
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem) + 2;  // x
    int* s_bounds = reinterpret_cast<int*>(smem + 32);       // CSR entries [p0, p1) of the CTA's rows
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.off_x);
    uint8_t* luts = smem + P.off_lut;
    float* s_head = reinterpret_cast<float*>(smem + P.off_head);
    float* s_tail = reinterpret_cast<float*>(smem + P.off_tail);
    int* s_headrow = reinterpret_cast<int*>(smem + P.off_headrow);
    int* s_tailrow = reinterpret_cast<int*>(smem + P.off_tailrow);
    float* s_rowsum = reinterpret_cast<float*>(smem + P.off_rowsum);
    float* s_ctile = reinterpret_cast<float*>(smem + P.off_ctile);
    float* s_slots = reinterpret_cast<float*>(smem + P.off_slots);
    int* s_wrange = reinterpret_cast<int*>(smem + P.off_wrange);  // [warp] = {first unit, end unit, first tile}
    int* s_tinfo = reinterpret_cast<int*>(smem + P.off_tinfo);    // [tile] = {mask of warps holding parts}

    // ---- rows of the CTA's tiles and their outliers
    const int ra = min(p.n_out, t_first * kTileRows);
    const int nrows = min(p.n_out, t_end * kTileRows) - ra;
    const bool has_csr = p.nnz > 0 && nrows > 0;
    const int rp_off = ra & 3;

    // ---- barriers, warp ranges, per-tile contributor masks
    if (lane == 0) {
        s_wrange[warp * 3] = wu0;
        s_wrange[warp * 3 + 1] = wu1;
        s_wrange[warp * 3 + 2] = wfirst;
    }
    if (tid == 0) {
        mbar_init(lbar, 1);
        mbar_init(cbar, 1);
        mbar_init(xbar, 1);
    }
    for (int tl = tid; tl < ctiles; tl += kThreads) {
        const int ta_u = (t_first + tl) * nsg, tb_u = ta_u + nsg;
        // warps holding a part of the tile (a warp range may be empty when
        // the CTA has fewer units than warps)
        int mask = 0;
        for (int wv = 0; wv < kWarps; ++wv) {
            const int a = u0 + cn * wv / kWarps, b = u0 + cn * (wv + 1) / kWarps;
            if (max(a, ta_u) < min(b, tb_u)) mask |= 1 << wv;
        }
        s_tinfo[tl] = mask;
    }
    if (has_csr) {
        for (int i = tid; i < nrows * CM; i += kThreads) s_rowsum[i] = 0.f;
        s_headrow[tid] = -1;
        s_tailrow[tid] = -1;
    }
    fence_mbar_init();
    __syncthreads();

    // ---- weights that do not depend on the previous kernel: the LUT planes
    // of the CTA's tiles, then (after reading the CTA's rowptr bounds) its
    // CSR slices, which are only needed after the dense part
    if (tid == 0) {
        const uint32_t lut_bytes = (uint32_t)ctiles * kTileRows * F::kLutBytes;
        mbar_expect_tx(lbar, lut_bytes);
        bulk_g2s(luts, p.lutp + (int64_t)t_first * kTileRows * F::kLutBytes, lut_bytes, lbar);
        const int q0 = has_csr ? p.rowptr[ra] : 0, q1 = has_csr ? p.rowptr[ra + nrows] : 0;
        s_bounds[0] = q0;
        s_bounds[1] = q1;
        const int nzz = q1 - q0;
        const bool in_smem = has_csr && nzz <= kCsrCap;
        const uint32_t rp_bytes = has_csr ? (uint32_t)round_up(nrows + 1 + rp_off, 4) * 4 : 0u;
        const uint32_t col_bytes = in_smem ? (uint32_t)round_up(nzz + (q0 & 3), 4) * 4 : 0u;
        const uint32_t val_bytes = in_smem ? (uint32_t)round_up(nzz + (q0 & 7), 8) * 2 : 0u;
        mbar_expect_tx(cbar, rp_bytes + col_bytes + val_bytes);
        if (rp_bytes) bulk_g2s(smem + P.off_rp, p.rowptr + (ra - rp_off), rp_bytes, cbar);
        if (col_bytes) bulk_g2s(smem + P.off_col, p.col + (q0 - (q0 & 3)), col_bytes, cbar);
        if (val_bytes) bulk_g2s(smem + P.off_val, p.val + (q0 - (q0 & 7)), val_bytes, cbar);
    }

    // ---- x and y may be written or read by the previous kernel of the
    // stream: wait for it to finish
    pdl_wait_previous();
    if (tid == 0) {
        if (p.x_bulk) {
            mbar_expect_tx(xbar, (uint32_t)p.batch * p.k_in * 2);
            for (int b = 0; b < p.batch; ++b) bulk_g2s(xs + b * P.x_stride, p.x + b * p.ldx, p.k_in * 2, xbar);
        } else {
            mbar_expect_tx(xbar, 0);
        }
    }
    if (!p.x_bulk) {
        for (int i = tid; i < p.batch * p.k_in; i += kThreads) {
            const int b = i / p.k_in, k = i - b * p.k_in;
            xs[b * P.x_stride + k] = p.x[b * p.ldx + k];
        }
    }
    const bool got_l = mbar_wait(lbar, 0), got_x = mbar_wait(xbar, 0);
    const bool ok = __syncthreads_and(got_l && got_x ? 1 : 0) != 0;
    if (!ok && tid == 0) atomicOr(p.status, kStatusWaitTimeout);

    // ---- dense part
    const int B = p.batch;
    const int xrow = (g < B) ? g : 0;  // batch column of this lane's B fragment (n = g)
    const int xrow2 = (NT == 2 && g + 8 < B) ? g + 8 : 0;
    TAB tg, tg8;
    float d0[NT][4], d1[NT][4];
    float f0 = 0.f, f1 = 0.f;  // CUDA-core accumulators (rows g, g+8)
    int tile = -1;

    // Hand this warp's part of `tile` to the CTA (shared memory).
    auto flush_tile = [&]() {
        float rr[NT][4];
        if constexpr (TC) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) rr[n][q] = d0[n][q] + d1[n][q];
        } else {
            f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
            f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
            rr[0][0] = f0;
            rr[0][1] = 0.f;
            rr[0][2] = f1;
            rr[0][3] = 0.f;
        }
        const int tl = tile - t_first;
        const int mask = s_tinfo[tl];
        const bool excl = (mask & (mask - 1)) == 0;  // this warp is the tile's only contributor
        float* dst = excl ? s_ctile + tl * TE : s_slots + (warp * 2 + (tile == wfirst ? 0 : 1)) * TE;
        if constexpr (SB) {
            if (t4 == 0) {
                dst[g] = rr[0][0];
                dst[g + 8] = rr[0][2];
            }
        } else {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int col = 8 * n + 2 * t4;
                dst[g * CM + col] = rr[n][0];
                dst[g * CM + col + 1] = rr[n][1];
                dst[(g + 8) * CM + col] = rr[n][2];
                dst[(g + 8) * CM + col + 1] = rr[n][3];
            }
        }
    };

    // Decode and multiply-accumulate one unit (16 rows x 256 columns).
    auto process = [&](const uint4 (&v)[F::kVecs], int unit) {
        const int ut = unit / nsg;
        if (ut != tile) {
            if (tile >= 0) flush_tile();
            tile = ut;
            const uint8_t* lt = luts + (tile - t_first) * kTileRows * F::kLutBytes;
            if constexpr (BITS == 3) {
                tg = load_tab3(lt + g * F::kLutBytes);
                tg8 = load_tab3(lt + (g + 8) * F::kLutBytes);
            } else {
                tg = load_tab4(lt + g * F::kLutBytes);
                tg8 = load_tab4(lt + (g + 8) * F::kLutBytes);
            }
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) d0[n][q] = d1[n][q] = 0.f;
            f0 = f1 = 0.f;
        }
        uint32_t w[4 * F::kVecs];
#pragma unroll
        for (int m = 0; m < F::kVecs; ++m) w[4 * m] = v[m].x, w[4 * m + 1] = v[m].y, w[4 * m + 2] = v[m].z, w[4 * m + 3] = v[m].w;
        const int step0 = (unit - tile * nsg) * kSgSteps;
        const int nvalid = min(kSgSteps, p.nsteps - step0);
        // x fragment source: batch rows >= B read row 0 (those MMA columns
        // are never written out), so every lane loads unconditionally
        const uint16_t* xb0 = xs + xrow * P.x_stride + step0 * 16 + 4 * t4;
        const uint16_t* xb1 = xs + xrow2 * P.x_stride + step0 * 16 + 4 * t4;
        auto mac = [&](int st, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
            if constexpr (TC) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xb0 + st * 16);
                if (st & 1)
                    mma16816(d1[0], a0, a1, a2, a3, xv.x, xv.y);
                else
                    mma16816(d0[0], a0, a1, a2, a3, xv.x, xv.y);
                if constexpr (NT == 2) {
                    const uint2 xw = *reinterpret_cast<const uint2*>(xb1 + st * 16);
                    if (st & 1)
                        mma16816(d1[1], a0, a1, a2, a3, xw.x, xw.y);
                    else
                        mma16816(d0[1], a0, a1, a2, a3, xw.x, xw.y);
                }
            } else {
                const uint2 xv = *reinterpret_cast<const uint2*>(xb0 + st * 16);
                fma2_mixed(f0, a0, xv.x);
                fma2_mixed(f0, a2, xv.y);
                fma2_mixed(f1, a1, xv.x);
                fma2_mixed(f1, a3, xv.y);
            }
        };
        if (nvalid == kSgSteps) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if constexpr (BITS == 3) {
                    const uint32_t w0 = w[3 * q], w1 = w[3 * q + 1], w2 = w[3 * q + 2];
                    uint32_t a0, a1, a2, a3;
                    decode3(tg, tg8, w0 & 0x77777777u, a0, a1, a2, a3);
                    mac(4 * q, a0, a1, a2, a3);
                    decode3(tg, tg8, w1 & 0x77777777u, a0, a1, a2, a3);
                    mac(4 * q + 1, a0, a1, a2, a3);
                    decode3(tg, tg8, w2 & 0x77777777u, a0, a1, a2, a3);
                    mac(4 * q + 2, a0, a1, a2, a3);
                    decode3(tg, tg8, sel3_extra(w0, w1, w2), a0, a1, a2, a3);
                    mac(4 * q + 3, a0, a1, a2, a3);
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t a0, a1, a2, a3;
                        decode4(tg, tg8, w[4 * q + j], a0, a1, a2, a3);
                        mac(4 * q + j, a0, a1, a2, a3);
                    }
                }
            }
        } else {
            // ragged last super-group (K % 256 != 0): steps < nvalid only
#pragma unroll
            for (int st = 0; st < kSgSteps; ++st) {
                if (st < nvalid) {
                    uint32_t a0, a1, a2, a3;
                    decode_step<BITS>(tg, tg8, w, st, a0, a1, a2, a3);
                    mac(st, a0, a1, a2, a3);
                }
            }
        }
    };

    // Software pipeline over the warp's units: slot j holds unit base+j; it
    // is refilled with unit base+j+D as soon as its words are taken.
    for (int base = 0; base < nwu; base += D) {
#pragma unroll
        for (int j = 0; j < D; ++j) {
            const int i = base + j;
            if (i < nwu) {
                uint4 v[F::kVecs];
#pragma unroll
                for (int m = 0; m < F::kVecs; ++m) v[m] = R[j][m];
                if (i + D < nwu) {
                    const uint8_t* src = p.codes + (int64_t)(wu0 + i + D) * F::kSgBytes + lane * 16;
#pragma unroll
                    for (int m = 0; m < F::kVecs; ++m) R[j][m] = ldg_stream_u128(src + m * 512);
                }
                process(v, wu0 + i);
            }
        }
    }
    if (tile >= 0) flush_tile();

    // ---- sparse part: a fixed share of nonzeros per thread (balanced);
    // its slices were copied while the dense part ran
    const bool got_c = mbar_wait(cbar, 0);
    if (!got_c && lane == 0) atomicOr(p.status, kStatusWaitTimeout);
    const int* s_rp = reinterpret_cast<const int*>(smem + P.off_rp) + rp_off;
    const int p0 = s_bounds[0], p1 = s_bounds[1];
    const int nz = p1 - p0;
    const bool csr_smem = has_csr && nz <= kCsrCap;
    const int* csr_col = csr_smem ? reinterpret_cast<const int*>(smem + P.off_col) + (p0 & 3) - p0 : p.col;
    const uint16_t* csr_val =
        csr_smem ? reinterpret_cast<const uint16_t*>(smem + P.off_val) + (p0 & 7) - p0 : p.val;
    const int e_per = has_csr ? max(1, (nz + kCsrThreads - 1) / kCsrThreads) : 1;
    if (has_csr && got_c) {
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
            int nxt = s_rp[cur + 1];
            bool first = true;
            float acc[CM];
#pragma unroll
            for (int b = 0; b < CM; ++b) acc[b] = 0.f;
            auto emit = [&](bool last) {
                float* dstp;
                if (first) {
                    s_headrow[tid] = cur;
                    dstp = s_head + tid * CM;
                } else if (last) {
                    s_tailrow[tid] = cur;
                    dstp = s_tail + tid * CM;
                } else {
                    dstp = s_rowsum + cur * CM;
                }
#pragma unroll
                for (int b = 0; b < CM; ++b) dstp[b] = acc[b];
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
                    while (q >= nxt) {
                        emit(false);
                        first = false;
#pragma unroll
                        for (int b = 0; b < CM; ++b) acc[b] = 0.f;
                        ++cur;
                        nxt = s_rp[cur + 1];
                    }
#pragma unroll
                    for (int b = 0; b < CM; ++b)
                        if (SB || b < B) acc[b] = fmaf(vv[j], h2f(xs[b * P.x_stride + cc[j]]), acc[b]);
                }
            }
            emit(true);
        }
    }
    __syncthreads();  // every warp's dense parts and every sparse partial are in shared memory

    // ---- finish the CTA's tiles: sum the warps' parts in warp order, add
    // the rows' nonzeros (interior sums plus the pieces of the threads whose
    // shares cut a row, in thread order) and write y
    for (int idx = tid; idx < ctiles * TE; idx += kThreads) {
        const int tl = idx / TE, e = idx - tl * TE;
        const int tile_i = t_first + tl;
        const int row_l = e / CM, col = e - row_l * CM;
        const int mask = s_tinfo[tl];
        float sum;
        if ((mask & (mask - 1)) == 0) {
            sum = s_ctile[idx];
        } else {
            sum = 0.f;
            for (int mm = mask; mm; mm &= mm - 1) {
                const int wv = __ffs(mm) - 1;
                sum += s_slots[(wv * 2 + (tile_i == s_wrange[wv * 3 + 2] ? 0 : 1)) * TE + e];
            }
        }
        const int row = tile_i * kTileRows + row_l;
        if (has_csr && row < ra + nrows) {
            const int i = row - ra;
            const int rs = s_rp[i], re = s_rp[i + 1];
            float cs = s_rowsum[i * CM + col];
            if (re > rs) {
                const int tau_a = (rs - p0) / e_per, tau_b = min(kCsrThreads - 1, (re - 1 - p0) / e_per);
                for (int tau = tau_a; tau <= tau_b; ++tau) {
                    if (s_headrow[tau] == i) cs += s_head[tau * CM + col];
                    if (s_tailrow[tau] == i) cs += s_tail[tau * CM + col];
                }
            }
            sum += cs;
        }
        if (row < p.n_out && col < B) p.y[col * p.ldy + row] = f2h_rn(sum);
    }
}

}  // namespace tc
}  // namespace sqz
