// kernels_tc.cuh -- the fused Dense-and-Sparse GEMV for sm_100a.
//
// y = (Q + S) x ("SqueezeLLM: Dense-and-Sparse Quantization", summary page,
// §3.4 "Kernel Implementation": LUT-based dense kernel, balanced sparse
// kernel, both fused into one launch).
//
// Work decomposition
//   * Rows are grouped in tiles of 16 (the M of an m16n8k16 MMA); columns in
//     super-groups of 256 (16 k16-steps).  A unit = (tile, super-group).
//   * One CTA of 12 warps per SM and call; its registers and shared memory
//     fit two CTAs on an SM, so the next call's CTA (programmatic dependent
//     launch) is resident while this one computes.  Each CTA owns a
//     contiguous run of whole tiles (runs differ by at most one tile, or,
//     for skewed outliers, follow a split by weight that the layer computed
//     at creation: cta_tile_range) and its
//     warps split the CTA's units into contiguous ranges (equal, except that
//     the eight warps that also sum the sparse part give one unit each to the
//     other warps when the layer has outliers), so a tile is finished inside
//     one CTA: no global atomics, no second pass.
//   * A warp that holds a whole tile writes its rows of y itself.  Tiles
//     split between warps are finished after the dense loop: one CTA
//     barrier, then the threads add the warps' parts of every shared tile in
//     warp order (deterministic, the same order for every batch size), add
//     each row's sparse sum and write y.
//
// Streaming: every warp streams its units through a private ring of
// shared-memory stages with asynchronous 16-byte copies (cp.async, one
// commit group per unit), keeping stages-1 units in flight while it
// decodes.  The copies are asynchronous on purpose: the barriers of the
// prologue never wait for the code stream.  Before waiting for the previous
// kernel of the stream (programmatic dependent launch; the weights never
// depend on it) a CTA requests its LUT planes, rowptr slice and sparse
// entries (bulk copies) and the first code units of every warp; x is
// requested right after the wait and ahead of the remaining code units.
// Waits on the bulk copies are bounded and record a status bit instead of
// hanging.
//
// Decode (kernel-native code layout, built by repack_codes_kernel): for each
// k16-step a lane holds 4 codes of row g and 4 of row g+8 (g = lane/4) at
// columns 4*t4..4*t4+3 (t4 = lane%4) of the step.  A code indexes the row's
// LUT kept in registers as byte planes (low bytes, high bytes); `prmt`
// gathers the bytes of four weights at once and two more `prmt` interleave
// them into fp16 pairs, which are exactly the A fragment of the MMA once
// the MMA's k order is permuted to match (the same permutation is applied
// to x, so the product is unchanged).  The byte permutes run on the integer
// ALU pipe, which bounds the dense part.
//
// Padding instead of ragged paths: columns past K inside the last
// super-group carry, per row, the code of a finite LUT entry, and x is zero
// there in shared memory, so every unit is a full 16-step unit and the
// padded products are exact zeros.
//
// MAC: fp16 x fp16 products are exact in fp32; accumulation is fp32, on the
// tensor cores (mma.sync m16n8k16, batch columns in N), on the CUDA cores
// (mixed-precision fma.rn.f32.f16, batch 1) or split between both (even
// steps on the tensor cores, odd steps on the CUDA cores, batch 1).
//
// Sparse part: the CSR entries of the rows of a CTA's tiles are split evenly
// over 256 of its threads (a fixed number of nonzeros per thread,
// independent of how skewed the rows are) -- the balanced scheme of the
// pages.  Each thread sums its share per row (head piece, rows it holds
// whole, tail piece) after x has arrived and before its dense loop; after a
// barrier of those 256 threads, each row's interior sum and the pieces of the
// threads whose shares cut the row are added into the row's slot -- in
// thread order by one thread, or, for a row cut into more than kLongPieces
// shares, by a warp in a fixed order (deterministic either way) -- and the
// threads arrive on an mbarrier that the writers of y wait on.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace sqz {
namespace tc {

constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
// Two CTAs fit on an SM: while one call's CTA decodes, the next call's CTA
// (programmatic dependent launch) already streams its own weights in.
constexpr int kCtasPerSm = 2;
constexpr int kCsrThreads = 256;  // threads sharing the sparse part (warps 0-7; the same split for every batch)
constexpr int kCsrWarps = kCsrThreads / 32;
static_assert(kCsrWarps <= kWarps && kWarps <= 16, "the sparse part runs on the CTA's first warps; warp masks are 16 bits");
// Dense units that each sparse warp hands to a non-sparse warp when the
// layer has outliers: the sparse share delays a warp's dense start by about
// one unit's decode time.
constexpr int kCsrUnitShift = 1;
constexpr int kTileRows = 16;
constexpr int kSgSteps = 16;      // k16-steps per super-group
constexpr int kSgCols = 256;      // columns per super-group
constexpr int kMaxCtas = 512;     // CTAs per launch (one per SM)
constexpr int kMinStages = 2;     // shared-memory stages per warp (units in flight + 1)
constexpr int kMaxStages = 16;
constexpr int kRingStages = 4;    // ring depth reserved before the CSR staging area
constexpr int kSbStages = 4;      // one pass over K: the ring depth, 4 stages (3 when 4 do not fit),
                                  // so that the wait for a unit's copies is one of two fixed forms
constexpr int kPreWait = 2;       // code units per warp requested before waiting for the previous kernel;
                                  // the rest of the first ring follows once x has landed
constexpr int kCsrCap = 4096;     // CSR entries per CTA staged in shared memory, at most (more: read from global)
// A row whose nonzeros are cut into more than kLongPieces shares (a long
// row of skewed outliers spans up to every share of its CTA) has its pieces
// added by a whole warp instead of one thread walking them in order.
constexpr int kLongPieces = 16;
constexpr uint32_t kSuspendNs = 1000000u;  // 1 ms per poll
constexpr uint32_t kWaitLimit = 2000u;

constexpr int kStatusWaitTimeout = 1;

// Multiply-accumulate units (template argument MAC).
constexpr int kMacTensor = 0;
constexpr int kMacCuda = 1;
constexpr int kMacMixed = 2;

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
    int grid;        // CTAs
    int ctiles_max;  // max tiles owned by one CTA
    int x_stride;    // shared-memory row stride of x, in halves
    int x_cols;      // columns of x kept in a shared-memory buffer (chunk_sg * 256; zero past K)
    int passes;      // passes over K (1, or more when x is staged in K chunks)
    int chunk_sg;    // super-groups of x per pass
    int xbufs;       // x buffers (2 when passes > 1: the next chunk loads during a pass)
    int cm;          // batch columns carried by the sparse part and the combine (carried_columns)
    int stages;      // shared-memory stages of each warp's code ring
    int csr_cap;     // CSR entries of a CTA that are staged in shared memory (more: read from global)
    // byte offsets
    int off_x, off_lut, off_rp, off_rowsum, off_head, off_tail, off_headrow, off_tailrow, off_slots, off_wrange,
        off_tinfo, off_col, off_val, off_acc, off_ring, total;
};

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Batch columns a launch carries through the sparse part, the warps' slots
// and the combine: 1 for batch 1, else the batch rounded up to 2, 4 or 8
// (one n-tile) or 16 (two).  The MMA always computes 8 columns per n-tile;
// carrying fewer keeps the shared memory of batches 2-4 small enough for
// two CTAs per SM.
__host__ __device__ inline int carried_columns(int batch, int nt, bool single) {
    if (single) return 1;
    if (nt == 2) return 16;
    return batch <= 2 ? 2 : batch <= 4 ? 4 : 8;
}

// First tile of CTA c when `ntiles` tiles are split over `grid` CTAs: the
// first ntiles % grid CTAs take one tile more (32-bit arithmetic only).
__host__ __device__ inline int tile_begin(int ntiles, int grid, int c) {
    const int q = ntiles / grid, r = ntiles - q * grid;
    return c * q + (c < r ? c : r);
}

// First unit of warp w among a CTA's units [u0, u0 + cn): an even split,
// except that the sparse warps (0..kCsrWarps-1) give `shift` units each to
// the other warps (spread evenly over them).
__host__ __device__ inline int warp_unit_begin(int u0, int cn, int w, int shift) {
    if (cn < 4 * kWarps || kCsrWarps == kWarps) shift = 0;
    const int moved = kCsrWarps * shift;
    const int base = cn - moved;
    const int extra = w > kCsrWarps ? moved * (w - kCsrWarps) / (kWarps - kCsrWarps) : 0;
    return u0 + base * w / kWarps + extra;
}

// CTAs of a launch: one per SM, at most one per tile.
__host__ __device__ inline int grid_size(int n_out, int sms) {
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int g = ntiles < sms ? ntiles : sms;
    return g < 1 ? 1 : g;
}

// `budget`: shared memory a CTA may use.  After the fixed part, the code
// ring gets kMinStages stages per warp, the CSR staging area what is left up
// to kCsrCap entries, and the ring more stages (up to kMaxStages) from the
// rest; total > budget when not even kMinStages fit.
// `passes` > 1 stages x in K chunks of chunk_sg super-groups (two buffers)
// and keeps per-tile sums in shared memory between passes.
// `ctiles_max`: the most tiles one CTA owns (0: the even split's).
__host__ __device__ inline Plan make_plan(int bits, int n_out, int k_in, int batch, int nt, bool single, int sms,
                                          int budget, int passes = 1, int ctiles_max = 0) {
    Plan P{};
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int nsteps = (k_in + 15) / 16;
    const int nsg = (nsteps + kSgSteps - 1) / kSgSteps;
    const int lut_bytes = bits == 3 ? 16 : 32;
    P.grid = grid_size(n_out, sms);
    P.ctiles_max = (ntiles + P.grid - 1) / P.grid;
    if (ctiles_max > P.ctiles_max) P.ctiles_max = ctiles_max;
    P.cm = carried_columns(batch, nt, single);
    P.passes = passes < 1 ? 1 : (passes > nsg ? nsg : passes);
    P.chunk_sg = (nsg + P.passes - 1) / P.passes;
    P.passes = (nsg + P.chunk_sg - 1) / P.chunk_sg;
    P.xbufs = P.passes > 1 ? 2 : 1;
    P.x_cols = P.chunk_sg * kSgCols;
    // x rows: stride = 32 (mod 128) bytes keeps the batch rows of one
    // fragment load in different banks.
    const int xs_bytes = round_up(P.x_cols * 2, 128) + 32;
    P.x_stride = xs_bytes / 2;
    const int rows = P.ctiles_max * kTileRows;
    int off = 128;  // two mbarriers
    P.off_x = off;
    off += P.xbufs * round_up(batch * xs_bytes, 128);
    P.off_lut = off;
    off += round_up(rows * lut_bytes, 128);
    P.off_rp = off;
    off += round_up((rows + 8) * 4, 128);
    P.off_rowsum = off;
    off += round_up(rows * P.cm * 4, 128);
    // the sparse pieces of the threads and the warps' parts of shared tiles
    const int ct = kCsrThreads;
    P.off_head = off;
    P.off_tail = off + ct * P.cm * 4;
    P.off_headrow = P.off_tail + ct * P.cm * 4;
    P.off_tailrow = P.off_headrow + ct * 4;
    off += round_up(2 * ct * P.cm * 4 + 2 * ct * 4, 128);
    P.off_slots = off;
    off += round_up(kWarps * 2 * kTileRows * P.cm * 4, 128);
    P.off_wrange = off;
    off += round_up(kWarps * 3 * 4, 16);
    P.off_tinfo = off;
    off += round_up(P.ctiles_max * 4, 16);
    off = round_up(off, 128);
    P.off_acc = off;  // per-tile sums across passes
    if (P.passes > 1) off += round_up(rows * P.cm * 4, 128);
    const int sg_bytes = bits == 3 ? 1536 : 2048;
    // the CSR staging area takes what is left after a ring of kRingStages
    // (up to kCsrCap entries; entries beyond it are read from global memory)
    // batch 1: a ring of kSbStages stages when it fits beside at least a
    // small CSR stage, else one stage less
    const bool fixed = P.passes == 1;  // one pass: a ring of fixed depth (compile-time waits)
    int sb_stages = kSbStages;
    if (fixed && budget - off - kSbStages * kWarps * sg_bytes - 512 < 6 * 256) sb_stages = kSbStages - 1;
    const int ring_min = (fixed ? sb_stages : kRingStages) * kWarps * sg_bytes;
    int cap = (budget - off - ring_min - 512) / 6;  // 4-byte column + 2-byte value per entry
    cap = cap > kCsrCap ? kCsrCap : cap;
    P.csr_cap = cap < 0 ? 0 : cap & ~7;
    P.off_col = off;  // a slice starts up to 3 entries early and is rounded up to 4
    off += round_up((P.csr_cap + 8) * 4, 128);
    P.off_val = off;  // up to 7 entries early, rounded up to 8
    off += round_up((P.csr_cap + 16) * 2, 128);
    P.off_ring = off;
    int stages = (budget - off) / (kWarps * sg_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < kMinStages) stages = kMinStages;
    if (fixed) stages = sb_stages;
    P.stages = stages;
    off += stages * kWarps * sg_bytes;
    P.total = off;
    return P;
}

// The fields read first sit together at the start (parameter reads that
// miss the constant cache are slow at kernel start).
struct Params {
    const uint8_t* codes;    // [ntiles][nsg][sg_bytes], kernel-native layout
    int n_out, k_in, nsg, ntiles, batch;
    int has_csr;             // the layer has outliers
    int x_bulk;              // 1: every x row is 16-byte aligned -> bulk copies
    Plan plan;
    const uint8_t* lutp;     // [ntiles*16][lut_bytes], byte planes
    const int32_t* rowptr;   // canonical CSR (device copies owned by the layer)
    const int32_t* col;
    const uint16_t* val;
    const uint16_t* x;
    int64_t ldx;
    uint16_t* y;
    int64_t ldy;
    int* status;             // error bits (bounded waits that gave up)
    // CSR entries of the rows of CTA c: [csr_cta[c], csr_cta[c+1]) (device
    // array of grid + 1 values; all zero when the layer has no outliers).  Kept
    // out of the parameters: a small parameter block stays in the constant
    // cache, whose misses cost hundreds of cycles wherever a field is reread.
    const int32_t* csr_cta;
    // First tile of CTA c: cta_tiles[c] (grid + 1 values) when the layer's
    // outliers are skewed enough for a split by weight (tiles + nonzeros);
    // nullptr: the even split of tile_begin.
    const int32_t* cta_tiles;
};

// Tiles [first, end) of CTA c.
__device__ __forceinline__ void cta_tile_range(const int32_t* cta_tiles, int ntiles, int grid, int c, int& first,
                                               int& end) {
    if (cta_tiles) {
        first = __ldg(cta_tiles + c);
        end = __ldg(cta_tiles + c + 1);
    } else {
        first = tile_begin(ntiles, grid, c);
        end = tile_begin(ntiles, grid, c + 1);
    }
}

// ------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Arrive (release at CTA scope: the thread's earlier shared-memory writes are
// visible to a thread whose wait on this phase succeeds).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
// Asynchronous 16-byte global -> shared copy (L2 only), its commit group and
// the wait for all but the newest n groups of this thread.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_newest(int n) {
    switch (n) {
#define SQZ_WAIT_CASE(k) \
    case k: cp_async_wait<k>(); break;
        SQZ_WAIT_CASE(0) SQZ_WAIT_CASE(1) SQZ_WAIT_CASE(2) SQZ_WAIT_CASE(3) SQZ_WAIT_CASE(4) SQZ_WAIT_CASE(5)
        SQZ_WAIT_CASE(6) SQZ_WAIT_CASE(7) SQZ_WAIT_CASE(8) SQZ_WAIT_CASE(9) SQZ_WAIT_CASE(10) SQZ_WAIT_CASE(11)
        SQZ_WAIT_CASE(12) SQZ_WAIT_CASE(13)
#undef SQZ_WAIT_CASE
        default: cp_async_wait<14>(); break;
    }
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

// Four 3-bit codes in the low four nibbles of sel (bit 3 of each nibble
// clear; bits 16..31 are ignored by prmt) -> fp16 pairs (w0,w1), (w2,w3).
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

// 3-bit quad: a lane's words w0, w1, w2 hold the codes of steps 4q, 4q+1,
// 4q+2 in bits 0..2 of their nibbles; bit 3 of nibble n of word j is bit j
// of the step-(4q+3) code at nibble n.  Low 16 bits: row g; high: row g+8.
__device__ __forceinline__ uint32_t sel3_main(uint32_t w) { return w & 0x77777777u; }
__device__ __forceinline__ uint32_t sel3_extra(uint32_t w0, uint32_t w1, uint32_t w2) {
    return ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
}

// Decode one k16-step of a lane: a0/a2 = row g pairs, a1/a3 = row g+8 pairs.
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

// Step `st` (0..15) of a lane's super-group words (dequant export).
template <int BITS, class TAB>
__device__ __forceinline__ void decode_step(const TAB& tg, const TAB& tg8, const uint32_t* w, int st, uint32_t& a0,
                                            uint32_t& a1, uint32_t& a2, uint32_t& a3) {
    if constexpr (BITS == 3) {
        const int q = st >> 2, j = st & 3;
        const uint32_t m = j < 3 ? sel3_main(w[3 * q + j]) : sel3_extra(w[3 * q], w[3 * q + 1], w[3 * q + 2]);
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

// The sparse pieces of row i held by shares [tau_a, tau_b] (a head piece
// where the share's first row is i, a tail piece where its last row is),
// added by the 32 lanes of a warp: lane l sums shares tau_a + l, + 32, ...
// in order, then a fixed shuffle tree brings the lanes' sums to lane 0,
// which adds them to the row's interior sum.  The order depends only on the
// split of the nonzeros into shares, never on the batch size.
template <int CM>
__device__ __forceinline__ void add_long_row_pieces(int i, int tau_a, int tau_b, int lane, float* s_rowsum,
                                                    const int* s_headrow, const float* s_head,
                                                    const int* s_tailrow, const float* s_tail) {
    float part[CM];
#pragma unroll
    for (int b = 0; b < CM; ++b) part[b] = 0.f;
    for (int tau = tau_a + lane; tau <= tau_b; tau += 32) {
        if (s_headrow[tau] == i) {
#pragma unroll
            for (int b = 0; b < CM; ++b) part[b] += s_head[tau * CM + b];
        }
        if (s_tailrow[tau] == i) {
#pragma unroll
            for (int b = 0; b < CM; ++b) part[b] += s_tail[tau * CM + b];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int b = 0; b < CM; ++b) part[b] += __shfl_down_sync(0xffffffffu, part[b], off);
    if (lane == 0) {
#pragma unroll
        for (int b = 0; b < CM; ++b) s_rowsum[i * CM + b] += part[b];
    }
}

// Long rows of rows [0, nrows): warp w of the nw warps that call this scans
// rows w*32 + lane, + nw*32, ... and adds the pieces of each long row with
// the whole warp.  Warp-uniform: every lane of the calling warps enters.
template <int CM>
__device__ __forceinline__ void add_long_rows(int nrows, int warp, int nw, int lane, const int* s_rp, int q0,
                                              int e_per, int nshares, float* s_rowsum, const int* s_headrow,
                                              const float* s_head, const int* s_tailrow, const float* s_tail) {
    for (int i0 = warp * 32; i0 < nrows; i0 += nw * 32) {
        const int i = i0 + lane;
        int ta = 0, tb = -1;
        if (i < nrows) {
            const int rs = s_rp[i], re = s_rp[i + 1];
            if (re > rs) {
                ta = (rs - q0) / e_per;
                tb = min(nshares - 1, (re - 1 - q0) / e_per);
            }
        }
        unsigned int m = __ballot_sync(0xffffffffu, tb - ta >= kLongPieces);
        while (m) {
            const int l = __ffs(m) - 1;
            m &= m - 1;
            const int a = __shfl_sync(0xffffffffu, ta, l), b = __shfl_sync(0xffffffffu, tb, l);
            add_long_row_pieces<CM>(i0 + l, a, b, lane, s_rowsum, s_headrow, s_head, s_tailrow, s_tail);
        }
    }
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

// Code stored for the columns past K of a row: an entry whose value is
// finite, so that its product with the zero x there is an exact zero.
template <int BITS>
__device__ __forceinline__ uint32_t pad_code(const uint16_t* lut, int row) {
    constexpr int L = 1 << BITS;
    for (int e = 0; e < L; ++e)
        if ((lut[(int64_t)row * L + e] & 0x7c00u) != 0x7c00u) return (uint32_t)e;
    return 0u;
}

// One thread per output word of the kernel-native layout.
template <int BITS>
__global__ void repack_codes_kernel(const uint32_t* __restrict__ canon, const uint16_t* __restrict__ lut,
                                    int32_t n_out, int32_t k_in, int nsg, int64_t total_words,
                                    uint32_t* __restrict__ out) {
    using F = Fmt<BITS>;
    const int64_t wpr = (int64_t)k_in * BITS / 32;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < total_words;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t unit = wi / (F::kVecs * 128);
        const int rem = (int)(wi % (F::kVecs * 128));
        const int m = rem >> 7, lane = (rem >> 2) & 31, e = rem & 3;
        const int lw = 4 * m + e;  // word index within the lane's list
        const int tile = (int)(unit / nsg), sg = (int)(unit % nsg);
        const int g = lane >> 2, t4 = lane & 3;
        auto code_of = [&](int n, int step) -> uint32_t {
            const int row = tile * kTileRows + g + 8 * (n >> 2);
            if (row >= n_out) return 0u;  // padding rows: their LUT rows are zero
            const int k = (sg * kSgSteps + step) * 16 + 4 * t4 + (n & 3);
            if (k >= k_in) return pad_code<BITS>(lut, row);
            return canon_code<BITS>(canon, wpr, row, k);
        };
        uint32_t word = 0;
        if constexpr (BITS == 4) {
            for (int n = 0; n < 8; ++n) word |= code_of(n, lw) << (4 * n);
        } else {
            const int q = lw / 3, j = lw % 3;
            for (int n = 0; n < 8; ++n) {
                const uint32_t c = code_of(n, 4 * q + j);
                const uint32_t x = (code_of(n, 4 * q + 3) >> j) & 1u;
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

// CSR entry range of each CTA's rows: out[c] = rowptr[first row of CTA c],
// c = 0..grid (the last value is rowptr[n_out]).
__global__ void csr_cta_bounds_kernel(const int32_t* __restrict__ rowptr, const int32_t* __restrict__ cta_tiles,
                                      int32_t n_out, int ntiles, int grid, int32_t* __restrict__ out) {
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c <= grid; c += gridDim.x * blockDim.x) {
        const int64_t r = (int64_t)(cta_tiles ? cta_tiles[c] : tile_begin(ntiles, grid, c)) * kTileRows;
        out[c] = rowptr[r < n_out ? r : n_out];
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
            uint32_t a0, a1, a2, a3;
            decode_step<BITS>(tg, tg8, w, st, a0, a1, a2, a3);
            const int k = (sg * kSgSteps + st) * 16 + 4 * t4;  // columns k..k+3 (k_in is a multiple of 8)
            if (k >= k_in) continue;
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
// MAC: kMacTensor / kMacCuda / kMacMixed.  SB: batch 1 (one column carried
// through the sparse part and the combine).  CMX: the batch columns carried
// (the plan's cm, carried_columns); it equals the launch's batch rounded up.
template <int BITS, int NT, int MAC, bool SB, bool RW, int CMX = (SB ? 1 : 8 * NT)>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) gemv_fused_kernel(const __grid_constant__ Params p) {
    using F = Fmt<BITS>;
    using TAB = typename std::conditional<BITS == 3, Tab3, Tab4>::type;
    constexpr int BM = 8 * NT;              // batch columns of the MMA accumulators
    constexpr int CM = CMX;                 // batch columns carried after the dense loop
    static_assert(SB ? CMX == 1 : (CMX % 2 == 0 && CMX >= 2 && CMX <= BM && (NT == 1 || CMX > 8)),
                  "carried columns: 1 for batch 1, else an even count within the n-tiles");
    constexpr int TE = kTileRows * CM;      // elements of one tile's result
    constexpr int V = F::kVecs;
    constexpr int CT = kCsrThreads;
    static_assert(!SB || NT == 1, "single-batch variant uses one n-tile");
    static_assert(MAC == kMacTensor || SB, "CUDA-core multiply-accumulates carry one batch column");
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan& P = p.plan;

    // The next kernel in the stream may start as soon as SMs free up.
    pdl_launch_dependents();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int G = gridDim.x, c = blockIdx.x;
    const int nsg = p.nsg;
    int t_first, t_end;
    cta_tile_range(p.cta_tiles, p.ntiles, G, c, t_first, t_end);
    const int ctiles = t_end - t_first;
    const int u0 = t_first * nsg, cn = ctiles * nsg;  // the CTA's units: [u0, u0 + cn)
    const int shift = p.has_csr ? kCsrUnitShift : 0;
    const int wu0 = warp_unit_begin(u0, cn, warp, shift), wu1 = warp_unit_begin(u0, cn, warp + 1, shift);
    const int nwu = wu1 - wu0;
    const int wfirst = nwu > 0 ? wu0 / nsg : -1;  // first tile of this warp

    // ---- rows of the CTA's tiles (their CSR entry range is read where it
    // is used: an indexed parameter load takes long, and nothing before the
    // wait for x needs it except the copy of the CSR slices)
    const int ra = min(p.n_out, t_first * kTileRows);
    const int nrows = min(p.n_out, t_end * kTileRows) - ra;
    const bool layer_csr = p.has_csr != 0;

    uint64_t* lbar = reinterpret_cast<uint64_t*>(smem);      // LUT planes + rowptr slice
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem) + 1;  // x
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem) + 2;  // CSR slices
    uint64_t* rbar = reinterpret_cast<uint64_t*>(smem) + 3;  // sparse pieces written (CT arrivals)
    uint64_t* xbar1 = reinterpret_cast<uint64_t*>(smem) + 4;  // second x buffer (several passes)
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.off_x);
    const int PS = SB ? 1 : P.passes, CS = P.chunk_sg;  // batch 1 always takes one pass
    const int xbuf_h = round_up(p.batch * P.x_stride * 2, 128) / 2;  // halves per x buffer
    uint8_t* luts = smem + P.off_lut;
    float* s_rowsum = reinterpret_cast<float*>(smem + P.off_rowsum);
    float* s_head = reinterpret_cast<float*>(smem + P.off_head);
    float* s_tail = reinterpret_cast<float*>(smem + P.off_tail);
    int* s_headrow = reinterpret_cast<int*>(smem + P.off_headrow);
    int* s_tailrow = reinterpret_cast<int*>(smem + P.off_tailrow);
    float* s_slots = reinterpret_cast<float*>(smem + P.off_slots);
    int* s_wrange = reinterpret_cast<int*>(smem + P.off_wrange);  // [warp] = {first unit, end unit, first tile}
    int* s_tinfo = reinterpret_cast<int*>(smem + P.off_tinfo);    // [tile] = mask of warps holding parts
    const int rp_off = ra & 3;
    const int* s_rp = reinterpret_cast<const int*>(smem + P.off_rp) + rp_off;  // s_rp[i] = rowptr[ra + i]

    // ---- weights, independent of the previous kernel: LUT planes of the
    // CTA's tiles, the rowptr slice and the CSR entries of its rows
    if (tid == 0) {
        mbar_init(lbar, 1);
        mbar_init(xbar, 1);
        mbar_init(cbar, 1);
        mbar_init(rbar, CT);
        mbar_init(xbar1, 1);
        fence_mbar_init();
        const uint32_t lut_bytes = (uint32_t)ctiles * kTileRows * F::kLutBytes;
        const uint32_t rp_bytes = layer_csr ? (uint32_t)round_up(nrows + 1 + rp_off, 4) * 4 : 0u;
        mbar_expect_tx(lbar, lut_bytes + rp_bytes);
        bulk_g2s(luts, p.lutp + (int64_t)t_first * kTileRows * F::kLutBytes, lut_bytes, lbar);
        if (rp_bytes) bulk_g2s(smem + P.off_rp, p.rowptr + (ra - rp_off), rp_bytes, lbar);
        const int q0 = __ldg(p.csr_cta + c), nz = __ldg(p.csr_cta + c + 1) - q0;
        const bool csr_in_smem = nz > 0 && nz <= P.csr_cap;
        const uint32_t col_bytes = csr_in_smem ? (uint32_t)round_up(nz + (q0 & 3), 4) * 4 : 0u;
        const uint32_t val_bytes = csr_in_smem ? (uint32_t)round_up(nz + (q0 & 7), 8) * 2 : 0u;
        mbar_expect_tx(cbar, col_bytes + val_bytes);
        if (col_bytes) bulk_g2s(smem + P.off_col, p.col + (q0 - (q0 & 3)), col_bytes, cbar);
        if (val_bytes) bulk_g2s(smem + P.off_val, p.val + (q0 - (q0 & 7)), val_bytes, cbar);
    }

    // ---- this warp's code ring: unit wu0+i goes to stage i % S; one commit
    // group per unit (empty past the warp's range) keeps the group count
    // uniform.  Each lane copies and later reads only its own 16-byte
    // pieces (coalesced: a warp-wide copy covers 512 consecutive bytes).
    const int S = P.stages, D = S - 1;
    uint8_t* ring = smem + P.off_ring + warp * S * F::kSgBytes + lane * 16;
    // Several passes over K: pass q covers super-groups [q*CS, q*CS + cs(q)) of
    // every tile of the CTA; its ctiles*cs(q) units are split evenly over the
    // warps.  One pass: the warp's units are [wu0, wu1).
    auto pass_cs = [&](int q) { return min(CS, nsg - q * CS); };
    auto prange = [&](int q, int w, int& a, int& b) {
        const int n = ctiles * pass_cs(q);
        a = n * w / kWarps;
        b = n * (w + 1) / kWarps;
    };
    auto pass_unit = [&](int q, int j) {
        const int cs = pass_cs(q), tl = j / cs;
        return (t_first + tl) * nsg + q * CS + (j - tl * cs);
    };
    // producer cursor over this warp's unit sequence (all passes in order)
    int pq = 0, pj = wu0 - u0, pend = wu1 - u0;
    if (PS > 1) {
        prange(0, warp, pj, pend);
        while (pj >= pend && ++pq < PS) prange(pq, warp, pj, pend);
    }
    auto issue = [&](int stage) {
        if (pq < PS) {
            const int unit = PS == 1 ? u0 + pj : pass_unit(pq, pj);
            const uint8_t* src = p.codes + (int64_t)unit * F::kSgBytes + lane * 16;
            uint8_t* dst = ring + stage * F::kSgBytes;
#pragma unroll
            for (int m = 0; m < V; ++m) cp_async16(dst + m * 512, src + m * 512);
            ++pj;
            while (pj >= pend && ++pq < PS) prange(pq, warp, pj, pend);
        }
        cp_async_commit();
    };
    const int pre = D < kPreWait ? D : kPreWait;
    for (int j = 0; j < pre; ++j) issue(j);

    // ---- bookkeeping: warp ranges, contributors per tile, zeroed sparse
    // sums, zero x past K
    if (lane == 0) {
        s_wrange[warp * 3] = wu0;
        s_wrange[warp * 3 + 1] = wu1;
        s_wrange[warp * 3 + 2] = wfirst;
    }
    for (int tl = tid; tl < ctiles; tl += kThreads) {
        const int ta_u = (t_first + tl) * nsg, tb_u = ta_u + nsg;
        int mask = 0;
        for (int wv = 0; wv < kWarps; ++wv) {
            const int a = warp_unit_begin(u0, cn, wv, shift), b = warp_unit_begin(u0, cn, wv + 1, shift);
            if (max(a, ta_u) < min(b, tb_u)) mask |= 1 << wv;
        }
        s_tinfo[tl] = mask;
    }
    if (layer_csr) {
        for (int i = tid; i < nrows * CM; i += kThreads) s_rowsum[i] = 0.f;
        if (tid < CT) {
            s_headrow[tid] = -1;
            s_tailrow[tid] = -1;
        }
    }
    const int B = p.batch;
    // columns of x chunk q (the last one may be short; its buffer is zero past K)
    auto chunk_len = [&](int q) { return min(CS * kSgCols, p.k_in - q * CS * kSgCols); };
    auto zero_pad = [&](int q) {
        uint16_t* xb = xs + (q & 1) * xbuf_h;
        const int len = chunk_len(q), pad = P.x_cols - len;
        for (int i = tid; i < B * pad; i += kThreads) {
            const int b = i / pad;
            xb[b * P.x_stride + len + (i - b * pad)] = 0;
        }
    };
    if (PS <= 2) zero_pad(PS - 1);
    if (PS > 1)
        for (int i = tid; i < ctiles * TE; i += kThreads) reinterpret_cast<float*>(smem + P.off_acc)[i] = 0.f;
    __syncthreads();

    // ---- the CTA's CSR entries [q0, q1), a fixed share e_per per thread
    const int q0 = __ldg(p.csr_cta + c), q1 = __ldg(p.csr_cta + c + 1);
    const int nz = q1 - q0;
    const bool has_csr = nz > 0;
    const bool csr_in_smem = has_csr && nz <= P.csr_cap;
    const int e_per = has_csr ? (int)(((int64_t)nz + CT - 1) / CT) : 1;
    const int ca = tid < CT ? (int)min((int64_t)q1, (int64_t)q0 + (int64_t)tid * e_per) : q1;
    const int cb = RW ? ca : (int)min((int64_t)q1, (int64_t)ca + e_per);  // row-wise: no shares
    const int* csr_col = csr_in_smem ? reinterpret_cast<const int*>(smem + P.off_col) + (q0 & 3) - q0 : p.col;
    const uint16_t* csr_val =
        csr_in_smem ? reinterpret_cast<const uint16_t*>(smem + P.off_val) + (q0 & 7) - q0 : p.val;
    // The part of a thread's sparse share that does not need x -- the row of
    // its first entry and its first entries -- is done before the wait for
    // the previous kernel, while that kernel still computes.
    int cur = 0, nxt = 0;
    int cc[8];
    uint32_t vh[8];
    bool got_early = true;
    if (has_csr && ca < cb) {
        got_early = mbar_wait(lbar, 0) && mbar_wait(cbar, 0);
        // row (relative to ra) containing entry ca: largest r with s_rp[r] <= ca
        int lo = 0, hi = nrows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_rp[mid] <= ca) lo = mid; else hi = mid - 1;
        }
        cur = lo;
        nxt = s_rp[cur + 1];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int q = ca + j;
            const bool in = q < cb;
            cc[j] = in ? csr_col[q] : 0;
            vh[j] = in ? (uint32_t)csr_val[q] : 0u;
        }
    }

    // ---- x may be written by the previous kernel of the stream: wait for it.
    // Before that, warp 1 asks L2 for x's lines (a hint that returns nothing:
    // a line the previous kernel writes later is updated in L2, so the copy
    // after the wait reads the new values either way), which hides the DRAM
    // latency when x was written earlier.
    if (warp == 1) {
        const int lines = (p.k_in * 2 + 127) / 128;
        for (int b = 0; b < B; ++b) {
            const char* xr = reinterpret_cast<const char*>(p.x + b * p.ldx);
            for (int l = lane; l < lines; l += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(xr + l * 128));
        }
    }
    pdl_wait_previous();
    // x chunk q into buffer q % 2: bulk copies issued by thread 0 (x rows
    // 16-byte aligned), or copied by all threads (then a barrier follows)
    auto load_chunk = [&](int q) {
        uint64_t* bar = (q & 1) ? xbar1 : xbar;
        uint16_t* xb = xs + (q & 1) * xbuf_h;
        const int k0 = q * CS * kSgCols, len = chunk_len(q);
        if (p.x_bulk) {
            if (tid == 0) {
                mbar_expect_tx(bar, (uint32_t)B * len * 2);
                for (int b = 0; b < B; ++b) bulk_g2s(xb + b * P.x_stride, p.x + b * p.ldx + k0, len * 2, bar);
            }
        } else {
            if (tid == 0) mbar_expect_tx(bar, 0);
            for (int i = tid; i < B * len; i += kThreads) {
                const int b = i / len, k = i - b * len;
                xb[b * P.x_stride + k] = p.x[b * p.ldx + k0 + k];
            }
        }
    };
    load_chunk(0);
    if (PS > 1) load_chunk(1);
    // Each thread waits for the copies itself (an mbarrier wait makes the
    // bulk-copied bytes visible to it); only x copied by the threads needs a
    // barrier.
    const bool got_l = mbar_wait(lbar, 0), got_x = mbar_wait(xbar, 0), got_c = mbar_wait(cbar, 0);
    if (!(got_l && got_x && got_c && got_early)) atomicOr(p.status, kStatusWaitTimeout);
    if (!p.x_bulk) __syncthreads();
    // ---- the rest of the first D units (after x, which they would delay)
    for (int j = pre; j < D; ++j) issue(j);

    // ---- sparse part: a fixed share of nonzeros per thread (balanced).
    // Each thread sums its entries per row: the first and last rows it
    // touches go to head/tail pieces, rows it holds entirely to s_rowsum;
    // the pieces are combined per row below, then the threads arrive on
    // rbar, which the writers of y wait on.
    if (has_csr && ca < cb) {
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
        for (int base = ca; base < cb; base += 8) {
            if (base != ca) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int q = base + j;
                    const bool in = q < cb;
                    cc[j] = in ? csr_col[q] : 0;
                    vh[j] = in ? (uint32_t)csr_val[q] : 0u;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int q = base + j;
                if (q >= cb) break;
                while (q >= nxt) {
                    emit(false);
                    first = false;
#pragma unroll
                    for (int b = 0; b < CM; ++b) acc[b] = 0.f;
                    ++cur;
                    nxt = s_rp[cur + 1];
                }
                const float v = h2f((uint16_t)vh[j]);
#pragma unroll
                for (int b = 0; b < CM; ++b)
                    if (SB || b < B) {
                        // x of column cc[j]: staged in shared memory, or (x in K chunks) from L2
                        const uint16_t xv = PS == 1 ? xs[b * P.x_stride + cc[j]] : __ldg(p.x + b * p.ldx + cc[j]);
                        acc[b] = fmaf(v, h2f(xv), acc[b]);
                    }
            }
        }
        emit(true);
    }
    // Row-wise mode (the plain CSR scheme, for comparison): no shares; thread
    // t sums the whole rows t, t + CT, ... of the CTA into s_rowsum, so the
    // tile finishers wait for the thread holding the longest row.
    if (RW && has_csr && tid < CT) {
        for (int i = tid; i < nrows; i += CT) {
            float acc[CM];
#pragma unroll
            for (int b = 0; b < CM; ++b) acc[b] = 0.f;
            for (int j = s_rp[i], je = s_rp[i + 1]; j < je; ++j) {
                const float v = h2f(csr_val[j]);
                const int cj = csr_col[j];
#pragma unroll
                for (int b = 0; b < CM; ++b)
                    if (SB || b < B) {
                        const uint16_t xv = PS == 1 ? xs[b * P.x_stride + cj] : __ldg(p.x + b * p.ldx + cj);
                        acc[b] = fmaf(v, h2f(xv), acc[b]);
                    }
            }
#pragma unroll
            for (int b = 0; b < CM; ++b) s_rowsum[i * CM + b] = acc[b];
        }
    }
    // Balanced mode: once every share is written (a barrier of the CT sparse
    // threads), each row's interior sum and the pieces of the threads whose
    // shares cut it are added into s_rowsum -- in thread order by one thread,
    // or by a warp for a row cut into more than kLongPieces shares -- so a
    // row's sparse sum is one shared-memory read wherever y is written.
    if (!RW && has_csr && tid < CT) {
        asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory");
        // thread tid takes rows tid, tid + CT, ...; the loop runs warp by warp
        // so that the long rows of a 32-row group can be handed to the warp
        for (int i0 = warp * 32; i0 < nrows; i0 += CT) {
            const int i = i0 + lane;
            int tau_a = 0, tau_b = -1;
            if (i < nrows) {
                const int rs = s_rp[i], re = s_rp[i + 1];
                if (re > rs) {
                    tau_a = (rs - q0) / e_per;
                    tau_b = min(CT - 1, (re - 1 - q0) / e_per);
                }
            }
            const bool long_row = tau_b - tau_a >= kLongPieces;
            if (tau_b >= tau_a && !long_row) {
                float cs[CM];
#pragma unroll
                for (int b = 0; b < CM; ++b) cs[b] = s_rowsum[i * CM + b];
                for (int tau = tau_a; tau <= tau_b; ++tau) {
                    if (s_headrow[tau] == i) {
#pragma unroll
                        for (int b = 0; b < CM; ++b) cs[b] += s_head[tau * CM + b];
                    }
                    if (s_tailrow[tau] == i) {
#pragma unroll
                        for (int b = 0; b < CM; ++b) cs[b] += s_tail[tau * CM + b];
                    }
                }
#pragma unroll
                for (int b = 0; b < CM; ++b) s_rowsum[i * CM + b] = cs[b];
            }
            for (unsigned int m = __ballot_sync(0xffffffffu, long_row); m; m &= m - 1) {
                const int l = __ffs(m) - 1;
                const int a = __shfl_sync(0xffffffffu, tau_a, l), b = __shfl_sync(0xffffffffu, tau_b, l);
                add_long_row_pieces<CM>(i0 + l, a, b, lane, s_rowsum, s_headrow, s_head, s_tailrow, s_tail);
            }
        }
    }
    if (has_csr && tid < CT) mbar_arrive(rbar);

    // The sparse sum of row ra+i, batch column col (complete once rbar's
    // first phase has completed).
    bool csr_ready = !has_csr;
    auto csr_row_sum = [&](int i, int col) -> float {
        if (!has_csr) return 0.f;
        if (!csr_ready) {
            if (!mbar_wait(rbar, 0)) atomicOr(p.status, kStatusWaitTimeout);
            csr_ready = true;
        }
        return s_rowsum[i * CM + col];
    };

    // ---- dense part
    const int xrow = (g < B) ? g : 0;  // batch column of this lane's B fragment (n = g)
    const int xrow2 = (NT == 2 && g + 8 < B) ? g + 8 : 0;
    TAB tg, tg8;
    float d0[NT][4], d1[NT][4];
    float f0 = 0.f, f1 = 0.f;  // CUDA-core accumulators (rows g, g+8)
    int tile = wfirst;
    int sg = wu0 - wfirst * nsg;

    auto start_tile = [&]() {
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
    };

    // y for (row, batch column) = dense value + the row's sparse sum.
    auto out = [&](int row, int col, float v) {
        if (row < p.n_out && col < B) p.y[col * p.ldy + row] = f2h_rn(v + csr_row_sum(row - ra, col));
    };

    // Hand this warp's part of `tile` over: written out directly when the
    // warp holds the whole tile, otherwise into its slot (the slots of shared
    // tiles are added in warp order after the loop).
    auto flush_tile = [&]() {
        float rr[NT][4];
        if constexpr (MAC != kMacCuda) {
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) rr[n][q] = d0[n][q] + d1[n][q];
        }
        if constexpr (MAC != kMacTensor) {
            f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
            f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
            f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
            if constexpr (MAC == kMacCuda) {
                rr[0][0] = f0;
                rr[0][2] = f1;
                rr[0][1] = rr[0][3] = 0.f;
            } else {
                rr[0][0] += f0;
                rr[0][2] += f1;
            }
        }
        const int tl = tile - t_first;
        const int row0 = tile * kTileRows;
        const int mask = s_tinfo[tl];
        if ((mask & (mask - 1)) == 0) {
            if constexpr (SB) {
                if (t4 == 0) {
                    out(row0 + g, 0, rr[0][0]);
                    out(row0 + g + 8, 0, rr[0][2]);
                }
            } else {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int col = 8 * n + 2 * t4;
                    out(row0 + g, col, rr[n][0]);
                    out(row0 + g, col + 1, rr[n][1]);
                    out(row0 + g + 8, col, rr[n][2]);
                    out(row0 + g + 8, col + 1, rr[n][3]);
                }
            }
            return;
        }
        float* dst = s_slots + (warp * 2 + (tile == wfirst ? 0 : 1)) * TE;
        if constexpr (SB) {
            if (t4 == 0) {
                dst[g] = rr[0][0];
                dst[g + 8] = rr[0][2];
            }
        } else {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int col = 8 * n + 2 * t4;  // even, like CM: col < CM covers col + 1
                if (col < CM) {
                    dst[g * CM + col] = rr[n][0];
                    dst[g * CM + col + 1] = rr[n][1];
                    dst[(g + 8) * CM + col] = rr[n][2];
                    dst[(g + 8) * CM + col + 1] = rr[n][3];
                }
            }
        }
        // shared tiles are combined after the loop (one CTA barrier)
    };

    // Decode and multiply-accumulate one unit (16 rows x 256 columns).
    auto process = [&](const uint4 (&v)[V], int sgi, const uint16_t* xbuf) {
        // x fragment source (super-group sgi of the x buffer): batch rows >= B
        // read row 0 (those MMA columns are never written out), so every lane
        // loads unconditionally
        const uint16_t* xb0 = xbuf + xrow * P.x_stride + sgi * kSgCols + 4 * t4;
        const uint16_t* xb1 = xbuf + xrow2 * P.x_stride + sgi * kSgCols + 4 * t4;
        auto mac = [&](int st, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
            const uint2 xv = *reinterpret_cast<const uint2*>(xb0 + st * 16);
            const bool on_tc = MAC == kMacTensor || (MAC == kMacMixed && (st & 1) == 0);
            if (on_tc) {
                const int chain = MAC == kMacTensor ? (st & 1) : ((st >> 1) & 1);
                if (chain)
                    mma16816(d1[0], a0, a1, a2, a3, xv.x, xv.y);
                else
                    mma16816(d0[0], a0, a1, a2, a3, xv.x, xv.y);
                if constexpr (NT == 2) {
                    const uint2 xw = *reinterpret_cast<const uint2*>(xb1 + st * 16);
                    if (chain)
                        mma16816(d1[1], a0, a1, a2, a3, xw.x, xw.y);
                    else
                        mma16816(d0[1], a0, a1, a2, a3, xw.x, xw.y);
                }
            } else {
                fma2_mixed(f0, a0, xv.x);
                fma2_mixed(f0, a2, xv.y);
                fma2_mixed(f1, a1, xv.x);
                fma2_mixed(f1, a3, xv.y);
            }
        };
        uint32_t w[4 * V];
#pragma unroll
        for (int m = 0; m < V; ++m) w[4 * m] = v[m].x, w[4 * m + 1] = v[m].y, w[4 * m + 2] = v[m].z, w[4 * m + 3] = v[m].w;
        if constexpr (BITS == 3) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t w0 = w[3 * q], w1 = w[3 * q + 1], w2 = w[3 * q + 2];
                const uint32_t m0 = sel3_main(w0), m1 = sel3_main(w1), m2 = sel3_main(w2);
                uint32_t a0, a1, a2, a3;
                decode3(tg, tg8, m0, a0, a1, a2, a3);
                mac(4 * q, a0, a1, a2, a3);
                decode3(tg, tg8, m1, a0, a1, a2, a3);
                mac(4 * q + 1, a0, a1, a2, a3);
                decode3(tg, tg8, m2, a0, a1, a2, a3);
                mac(4 * q + 2, a0, a1, a2, a3);
                decode3(tg, tg8, sel3_extra(w0, w1, w2), a0, a1, a2, a3);
                mac(4 * q + 3, a0, a1, a2, a3);
            }
        } else {
#pragma unroll
            for (int st = 0; st < kSgSteps; ++st) {
                uint32_t a0, a1, a2, a3;
                decode4(tg, tg8, w[st], a0, a1, a2, a3);
                mac(st, a0, a1, a2, a3);
            }
        }
    };


    // ---- several passes over K (x staged chunk by chunk): per pass, each
    // warp decodes its share of the pass's units; a tile's part that a warp
    // holds whole is added to the tile's sum at once, shared parts go to the
    // warps' slots and are added in warp order after a CTA barrier (the same
    // order every call); the next chunk of x then loads into the buffer the
    // pass used.  After the last pass the tile sums get their sparse sums and
    // are written out.
    if (!SB && PS > 1) {  // (batch 1 always takes one pass)
        float* s_acc = reinterpret_cast<float*>(smem + P.off_acc);
        int s_read = 0, s_fill = D;
        for (int q = 0; q < PS; ++q) {
            const int cs = pass_cs(q);
            int a, b;
            prange(q, warp, a, b);
            const uint16_t* xq = xs + (q & 1) * xbuf_h;
            if (!mbar_wait((q & 1) ? xbar1 : xbar, (uint32_t)((q >> 1) & 1))) atomicOr(p.status, kStatusWaitTimeout);
            int cur = -1;  // CTA-local tile of the accumulators
            auto flush_pass = [&]() {
                float rr[NT][4];
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int r = 0; r < 4; ++r) rr[n][r] = d0[n][r] + d1[n][r];
                const int lo = cur * cs, hi = lo + cs;
                const bool whole = a <= lo && b >= hi;
                float* dst = whole ? s_acc + cur * TE : s_slots + (warp * 2 + (cur == a / cs ? 0 : 1)) * TE;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int col = 8 * n + 2 * t4;
                    if (col >= CM) continue;  // columns past the carried ones are never written out
                    if (whole) {
                        dst[g * CM + col] += rr[n][0];
                        dst[g * CM + col + 1] += rr[n][1];
                        dst[(g + 8) * CM + col] += rr[n][2];
                        dst[(g + 8) * CM + col + 1] += rr[n][3];
                    } else {
                        dst[g * CM + col] = rr[n][0];
                        dst[g * CM + col + 1] = rr[n][1];
                        dst[(g + 8) * CM + col] = rr[n][2];
                        dst[(g + 8) * CM + col + 1] = rr[n][3];
                    }
                }
            };
#pragma unroll 1
            for (int j = a; j < b; ++j) {
                cp_async_wait_newest(D - 1);
                uint4 v[V];
                const uint8_t* src = ring + s_read * F::kSgBytes;
#pragma unroll
                for (int m = 0; m < V; ++m) v[m] = *reinterpret_cast<const uint4*>(src + m * 512);
                issue(s_fill);
                s_read = s_read + 1 == S ? 0 : s_read + 1;
                s_fill = s_fill + 1 == S ? 0 : s_fill + 1;
                const int tl = j / cs;
                if (tl != cur) {
                    if (cur >= 0) flush_pass();
                    cur = tl;
                    tile = t_first + tl;
                    start_tile();
                }
                process(v, j - tl * cs, xq);
            }
            if (cur >= 0) flush_pass();
            // per tile of this pass: the warps holding parts (bits 0-15) and
            // which of them used their second slot (bits 16-31)
            for (int tl = tid; tl < ctiles; tl += kThreads) {
                const int lo = tl * cs, hi = lo + cs;
                int info = 0;
                for (int w = 0; w < kWarps; ++w) {
                    int aw, bw;
                    prange(q, w, aw, bw);
                    if (max(aw, lo) < min(bw, hi)) info |= (1 << w) | ((tl == aw / cs ? 0 : 1) << (16 + w));
                }
                s_tinfo[tl] = info;
            }
            __syncthreads();
            // shared tiles of this pass: the parts, in warp order
            for (int idx = tid; idx < ctiles * TE; idx += kThreads) {
                const int tl = idx / TE, e = idx - tl * TE;
                const int info = s_tinfo[tl], mask = info & 0xffff;
                if ((mask & (mask - 1)) == 0) continue;  // one part: already added
                float sum = 0.f;
                for (int mm = mask; mm; mm &= mm - 1) {
                    const int w = __ffs(mm) - 1;
                    sum += s_slots[(w * 2 + ((info >> (16 + w)) & 1)) * TE + e];
                }
                s_acc[idx] += sum;
            }
            // chunk q+2 into the buffer this pass used
            if (q + 2 < PS) {
                if (q + 2 == PS - 1) zero_pad(q + 2);
                if (tid == 0) fence_proxy_async();
                load_chunk(q + 2);
            }
            __syncthreads();
        }
        for (int idx = tid; idx < ctiles * TE; idx += kThreads) {
            const int tl = idx / TE, e = idx - tl * TE;
            const int row_l = e / CM, col = e - row_l * CM;
            out((t_first + tl) * kTileRows + row_l, col, s_acc[idx]);
        }
        return;
    }

    // Units in order: wait for unit i's group, read its stage, refill the
    // stage freed by unit i-1 with unit i+D, decode.
    if (nwu > 0) start_tile();
    int s_read = 0, s_fill = D;
#pragma unroll 1
    for (int i = 0; i < nwu; ++i) {
        if (S == kSbStages)  // single-pass plans: 4 stages, or 3
            cp_async_wait<kSbStages - 2>();
        else
            cp_async_wait<kSbStages - 3>();
        uint4 v[V];
        const uint8_t* src = ring + s_read * F::kSgBytes;
#pragma unroll
        for (int m = 0; m < V; ++m) v[m] = *reinterpret_cast<const uint4*>(src + m * 512);
        issue(s_fill);
        s_read = s_read + 1 == S ? 0 : s_read + 1;
        s_fill = s_fill + 1 == S ? 0 : s_fill + 1;
        process(v, sg, xs);
        if (++sg == nsg || i + 1 == nwu) {
            flush_tile();
            if (i + 1 < nwu) {
                ++tile;
                sg = 0;
                start_tile();
            }
        }
    }
    // Tiles shared by several warps: once every warp has left the loop, the
    // warps' parts are added in warp order (the same order for every batch
    // size) and the rows get their sparse sums.
    __syncthreads();
    csr_ready = true;  // every sparse share was written before this barrier
    for (int idx = tid; idx < ctiles * TE; idx += kThreads) {
        const int tl = idx / TE, e = idx - tl * TE;
        const int mask = s_tinfo[tl];
        if ((mask & (mask - 1)) == 0) continue;  // one warp: already written
        const int row_l = e / CM, col = e - row_l * CM;
        float sum = 0.f;
        for (int mm = mask; mm; mm &= mm - 1) {
            const int wv = __ffs(mm) - 1;
            sum += s_slots[(wv * 2 + (t_first + tl == s_wrange[wv * 3 + 2] ? 0 : 1)) * TE + e];
        }
        out((t_first + tl) * kTileRows + row_l, col, sum);
    }
}

}  // namespace tc
}  // namespace sqz
