// kernels_pd.cuh -- the fused Dense-and-Sparse GEMV with weights decoded into
// tensor memory ahead of the activations (batches of 1..8 columns).
//
// y = (Q + S) x ("SqueezeLLM: Dense-and-Sparse Quantization", summary page,
// §3.4 "Kernel Implementation": LUT-based dense kernel, balanced sparse
// kernel, both fused into one launch).
//
// Why: a call cannot use x before the previous kernel of the stream has
// finished (programmatic dependent launch, griddepcontrol.wait), and on B200
// that wait returns about a microsecond after the previous grid's last CTA
// exits; x then takes a few hundred nanoseconds more to arrive.  The dense
// part's cost is the LUT decode (byte permutes on the integer pipe), and the
// decode needs only the codes and the LUTs -- never x.  So every warp decodes
// its first code units while it waits, and parks their MMA A fragments in
// tensor memory (TMEM: 256 KB per SM that this path would otherwise leave
// unused; a tcgen05.st of a quad of k16-steps is nearly free next to the
// decode).  When x lands the warp stops decoding ahead (it checks the x
// barrier before every quad, without blocking), runs the MMAs of the
// fragments it parked (tcgen05.ld + mma.sync, about a third of the cost of
// decoding), and then decodes the rest of its units as usual.
//
// Work decomposition
//   * Rows in tiles of 16 (the M of an m16n8k16 MMA), columns in
//     super-groups of 256 (16 k16-steps); a unit = (tile, super-group).  The
//     code layout and decoder are those of kernels_tc.cuh.
//   * A CTA owns a contiguous run of whole tiles (the even split, or the
//     split by weight of the layer's tile array for skewed outliers).  It has
//     NW dense warps (8: two CTAs per SM; 16: one CTA per SM, see Shape) and
//     one control warp.  Its units are split into 16 contiguous, equal ranges
//     ("virtual warps"); with NW = 8 a warp runs two adjacent ranges.
//   * The control warp requests the LUT planes, the rowptr slice and the
//     CSR entries of the CTA (bulk copies), asks L2 for the CTA's codes,
//     allocates TMEM, waits for the previous kernel and copies x in.
//   * Decoding ahead starts only once the SM's earlier CTAs of this kernel
//     have finished their dense loops (or x has arrived): see g_pd_looped.
//   * Sparse part (the balanced scheme): the CTA's nonzeros are split evenly
//     into 512 shares (two per thread with NW = 8).  Before x arrives a
//     thread finds the row of its first entry and loads its first entries;
//     once x is there it sums its share per row (head piece, rows it holds
//     whole, tail piece).  Warps in the first half run their shares before
//     their decode loop, the others after it.
//   * Every virtual warp stores its part of each tile it touches in shared
//     memory (one slot for a tile it holds whole, its own slots for the
//     first and last tiles it shares); after one CTA barrier the threads add
//     the parts in virtual-warp order and each row's sparse sum (the
//     interior sum plus the pieces of the shares that cut the row, in share
//     order) and write y once.  Every summation order is fixed and does not
//     depend on NW: results are bitwise reproducible, both shapes give the
//     same bits, and a column of a batch equals the batch-1 call on it.
//
// TMEM: dense warp w reaches the 32 lanes of quarter w % 4 (lane = the
// warp's lane); its columns are [(w / 4) * 128, +128) of its CTA's
// allocation: two units of 64 columns (a quad of 4 k16-steps = 16 columns of
// A fragments).  The control warp allocates the CTA's columns (256 with
// NW = 8, 512 with NW = 16) at the start and frees them after the last
// tcgen05.ld, on every path; the resident CTAs of an SM never ask for more
// than its 512 columns together, so no allocation waits on a CTA that waits
// for it.
//
// Every wait on a copy or mbarrier is bounded and records a status bit
// instead of hanging.
#pragma once

#include "kernels_tc.cuh"

namespace sqz {
namespace pd {

using tc::Fmt;
using tc::kSgCols;
using tc::kSgSteps;
using tc::kTileRows;
using tc::round_up;

// Two shapes of CTA (template argument NW, the dense warps):
//   NW = 8:  8 dense warps + the control warp, two CTAs per SM, each with half
//            the TMEM (256 columns): the next call's CTA is resident while
//            this one computes, so it loads its LUTs and first code units and
//            parks its first units in TMEM before the previous call ends.
//   NW = 16: 16 dense warps + the control warp, one CTA per SM with all 512
//            columns (for calls whose shared memory does not fit half an SM).
// Either way a warp parks at most two units (128 columns of its quarter), at
// most two CTAs of this kernel are resident on an SM, and together they never
// ask for more than the SM's 512 columns, so no allocation ever waits for a
// CTA that waits for it.
// The summation structure does not depend on the shape: a CTA's units are
// split into 16 contiguous ranges ("virtual warps", each with its own
// accumulators and its own slots for the tiles it shares) and its nonzeros
// into 512 equal shares; with NW = 8 a warp runs two adjacent ranges one
// after the other and two shares.  Both shapes give the same bits.
constexpr int kVWarps = 16;
constexpr int kVThreads = kVWarps * 32;
template <int NW>
struct Shape {
    static constexpr int kDenseWarps = NW;
    static constexpr int kCtrlWarp = NW;
    static constexpr int kThreads = (NW + 1) * 32;
    static constexpr int kCtasPerSm = NW == 8 ? 2 : 1;
    static constexpr int kTmemCols = NW == 8 ? 256 : 512;
    static constexpr int kRanges = kVWarps / NW;  // virtual warps per warp
    static constexpr int kMinSmem = NW == 8 ? 0 : 120 * 1024;  // NW = 16: more than half an SM
};
constexpr int kStages = 4;    // code ring stages per dense warp
constexpr int kPreUnits = 2;  // units per warp that can be parked in TMEM
constexpr int kCsrCap = 4096; // CSR entries per CTA staged in shared memory

struct Plan {
    int grid, ctiles_max, x_stride, cm, csr_cap;
    int off_taddr, off_x, off_lut, off_rp, off_rowsum, off_head, off_tail, off_headrow, off_tailrow, off_slots,
        off_tsum, off_tinfo, off_col, off_val, off_ring, total;
};

// Shared-memory plan of a launch; total > budget when it does not fit.
__host__ __device__ inline Plan make_plan(int bits, int n_out, int k_in, int batch, int sms, int budget, int nw,
                                          int ctiles_max = 0) {
    Plan P{};
    const int min_smem = nw == 8 ? Shape<8>::kMinSmem : Shape<16>::kMinSmem;
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int nsg = ((k_in + 15) / 16 + kSgSteps - 1) / kSgSteps;
    const int lut_bytes = bits == 3 ? 16 : 32;
    const int sg_bytes = bits == 3 ? 1536 : 2048;
    P.grid = tc::grid_size(n_out, sms);
    P.ctiles_max = (ntiles + P.grid - 1) / P.grid;
    if (ctiles_max > P.ctiles_max) P.ctiles_max = ctiles_max;
    P.cm = batch == 1 ? 1 : 8;
    // x rows: stride = 32 (mod 128) bytes keeps the batch rows of one
    // fragment load in different banks
    const int xs_bytes = round_up(nsg * kSgCols * 2, 128) + 32;
    P.x_stride = xs_bytes / 2;
    const int rows = P.ctiles_max * kTileRows;
    int off = 128;  // mbarriers
    P.off_taddr = 64;
    P.off_x = off;
    off += round_up(batch * xs_bytes, 128);
    P.off_lut = off;
    off += round_up(rows * lut_bytes, 128);
    P.off_rp = off;
    off += round_up((rows + 8) * 4, 128);
    P.off_rowsum = off;
    off += round_up(rows * P.cm * 4, 128);
    const int ct = kVThreads;
    P.off_head = off;
    P.off_tail = off + ct * P.cm * 4;
    P.off_headrow = P.off_tail + ct * P.cm * 4;
    P.off_tailrow = P.off_headrow + ct * 4;
    off += round_up(2 * ct * P.cm * 4 + 2 * ct * 4, 128);
    P.off_slots = off;
    off += round_up(kVWarps * 2 * kTileRows * P.cm * 4, 128);
    P.off_tsum = off;  // sums of the tiles a warp holds whole
    off += round_up(rows * P.cm * 4, 128);
    P.off_tinfo = off;
    off += round_up(P.ctiles_max * 4, 128);
    const int ring = kStages * nw * sg_bytes;
    int cap = (budget - off - ring - 512) / 6;
    cap = cap > kCsrCap ? kCsrCap : cap;
    P.csr_cap = cap < 0 ? 0 : cap & ~7;
    P.off_col = off;  // a slice starts up to 3 entries early and is rounded up to 4
    off += round_up((P.csr_cap + 8) * 4, 128);
    P.off_val = off;  // up to 7 entries early, rounded up to 8
    off += round_up((P.csr_cap + 16) * 2, 128);
    P.off_ring = off;
    off += ring;
    P.total = off < min_smem ? min_smem : off;
    return P;
}

struct Params {
    const uint8_t* codes;    // [ntiles][nsg][sg_bytes], kernel-native layout
    int n_out, k_in, nsg, ntiles, batch;
    int has_csr;
    int x_bulk;              // 1: every x row is 16-byte aligned -> bulk copies
    Plan plan;
    const uint8_t* lutp;     // [ntiles*16][lut_bytes] byte planes
    const int32_t* rowptr;
    const int32_t* col;
    const uint16_t* val;
    const uint16_t* x;
    int64_t ldx;
    uint16_t* y;
    int64_t ldy;
    int* status;
    const int32_t* csr_cta;  // [grid + 1]: CSR entry range of each CTA's rows
    const int32_t* cta_tiles;  // [grid + 1]: first tile of each CTA, or nullptr (the even split)
};

// ------------------------------------------------------- per-SM hand-over
// Decoding ahead pays only while the SM has nothing else to do: in a chain of
// calls the next call's CTA is resident long before the current one has
// finished its dense loop, and decoding then would only take integer issue
// from it.  So every CTA of this kernel takes a ticket from its SM's start
// counter and, once its dense warps are done, bumps its SM's "loop done"
// counter; a CTA starts decoding ahead once every CTA of this kernel that
// started on its SM before it has finished its dense loop (or once its x has
// arrived).  The counters are hints only: the wait ends on either condition
// and is bounded, and it never orders anything that results depend on.
constexpr int kSmSlots = 256;
__device__ unsigned int g_pd_started[kSmSlots];
__device__ unsigned int g_pd_looped[kSmSlots];
__device__ __forceinline__ unsigned int sm_id() {
    unsigned int r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}
__device__ __forceinline__ unsigned int ld_relaxed(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
constexpr int kGatePolls = 20000;  // x 256 ns: the gate gives up after about 5 ms

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc::smem_u32(dst)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 16 consecutive 32-bit columns of the warp's 32 lanes (one value per lane each)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// Wait for this thread's tcgen05.ld; the registers of `r` pass through the
// instruction so that no use of them can be scheduled before it (the load
// writes them asynchronously).
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16], uint32_t (&r2)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                   "+r"(r2[0]), "+r"(r2[1]), "+r"(r2[2]), "+r"(r2[3]), "+r"(r2[4]), "+r"(r2[5]), "+r"(r2[6]),
                   "+r"(r2[7]), "+r"(r2[8]), "+r"(r2[9]), "+r"(r2[10]), "+r"(r2[11]), "+r"(r2[12]), "+r"(r2[13]),
                   "+r"(r2[14]), "+r"(r2[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The A fragments of quad q (k16-steps 4q..4q+3) of a unit: a[4j..4j+3] =
// (a0, a1, a2, a3) of step 4q+j.
template <int BITS, class TAB>
__device__ __forceinline__ void decode_quad(const TAB& tg, const TAB& tg8, const uint32_t (&w)[4 * Fmt<BITS>::kVecs],
                                            int q, uint32_t (&a)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        tc::decode_step<BITS>(tg, tg8, w, 4 * q + j, a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
}

// ------------------------------------------------------------ main kernel
// SB: batch 1 (one column carried through the sparse part and the combine).
template <int BITS, bool SB, int NW>
__global__ void __launch_bounds__(Shape<NW>::kThreads, Shape<NW>::kCtasPerSm)
    gemv_pd_kernel(const __grid_constant__ Params p) {
    constexpr int kCtrlWarp = Shape<NW>::kCtrlWarp;
    constexpr int kThreads = Shape<NW>::kThreads, kTmemCols = Shape<NW>::kTmemCols;
    constexpr int RG = Shape<NW>::kRanges;
    using F = Fmt<BITS>;
    using TAB = typename std::conditional<BITS == 3, tc::Tab3, tc::Tab4>::type;
    constexpr int CM = SB ? 1 : 8;           // batch columns carried after the dense loop
    constexpr int TE = kTileRows * CM;       // elements of one tile's result
    constexpr int V = F::kVecs;
    constexpr int S = kStages, D = kStages - 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const Plan& P = p.plan;

    tc::pdl_launch_dependents();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const bool ctrl = warp == kCtrlWarp;
    const int G = gridDim.x, c = blockIdx.x;
    const int nsg = p.nsg;
    int t_first, t_end;
    tc::cta_tile_range(p.cta_tiles, p.ntiles, G, c, t_first, t_end);
    const int ctiles = t_end - t_first;
    const int u0 = t_first * nsg, cn = ctiles * nsg;
    // virtual warp v: units [vbeg(v), vbeg(v + 1)) of the CTA; dense warp w
    // runs virtual warps w*RG .. w*RG+RG-1, i.e. units [wu0, wu1)
    auto vbeg = [&](int v) { return u0 + cn * v / kVWarps; };
    const int wsel = ctrl ? 0 : warp;
    const int wu0 = vbeg(wsel * RG), wu1 = vbeg((wsel + 1) * RG);
    const int nwu = ctrl ? 0 : wu1 - wu0;
    const int wfirst = nwu > 0 ? wu0 / nsg : -1;
    const int ra = min(p.n_out, t_first * kTileRows);
    const int nrows = min(p.n_out, t_end * kTileRows) - ra;
    const bool layer_csr = p.has_csr != 0;

    uint64_t* lbar = reinterpret_cast<uint64_t*>(smem);      // LUT planes + rowptr slice
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem) + 1;  // x
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem) + 2;  // CSR slices
    uint32_t* s_taddr = reinterpret_cast<uint32_t*>(smem + P.off_taddr);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.off_x);
    uint8_t* luts = smem + P.off_lut;
    float* s_rowsum = reinterpret_cast<float*>(smem + P.off_rowsum);
    float* s_head = reinterpret_cast<float*>(smem + P.off_head);
    float* s_tail = reinterpret_cast<float*>(smem + P.off_tail);
    int* s_headrow = reinterpret_cast<int*>(smem + P.off_headrow);
    int* s_tailrow = reinterpret_cast<int*>(smem + P.off_tailrow);
    float* s_slots = reinterpret_cast<float*>(smem + P.off_slots);
    float* s_tsum = reinterpret_cast<float*>(smem + P.off_tsum);
    int* s_tinfo = reinterpret_cast<int*>(smem + P.off_tinfo);  // [tile] = mask of virtual warps holding parts
    const int rp_off = ra & 3;
    const int* s_rp = reinterpret_cast<const int*>(smem + P.off_rp) + rp_off;  // s_rp[i] = rowptr[ra + i]
    const int B = p.batch;

    // ---- control warp: barriers, copies of the weights (independent of the
    // previous kernel), the L2 prefetch of the CTA's codes, TMEM
    const unsigned int smslot = sm_id() % kSmSlots;
    unsigned int* s_ticket = reinterpret_cast<unsigned int*>(smem + P.off_taddr + 4);
    if (ctrl) {
        if (lane == 0) {
            *s_ticket = atomicAdd(&g_pd_started[smslot], 1u);
            tc::mbar_init(lbar, 1);
            tc::mbar_init(xbar, p.x_bulk ? 1 : 32);  // bulk: one expect_tx; else every lane after its stores
            tc::mbar_init(cbar, 1);
            tc::fence_mbar_init();
            const uint32_t lut_bytes = (uint32_t)ctiles * kTileRows * F::kLutBytes;
            const uint32_t rp_bytes = layer_csr ? (uint32_t)round_up(nrows + 1 + rp_off, 4) * 4 : 0u;
            tc::mbar_expect_tx(lbar, lut_bytes + rp_bytes);
            tc::bulk_g2s(luts, p.lutp + (int64_t)t_first * kTileRows * F::kLutBytes, lut_bytes, lbar);
            if (rp_bytes) tc::bulk_g2s(smem + P.off_rp, p.rowptr + (ra - rp_off), rp_bytes, lbar);
            const int q0 = __ldg(p.csr_cta + c), nz = __ldg(p.csr_cta + c + 1) - q0;
            const bool csr_in_smem = nz > 0 && nz <= P.csr_cap;
            const uint32_t col_bytes = csr_in_smem ? (uint32_t)round_up(nz + (q0 & 3), 4) * 4 : 0u;
            const uint32_t val_bytes = csr_in_smem ? (uint32_t)round_up(nz + (q0 & 7), 8) * 2 : 0u;
            tc::mbar_expect_tx(cbar, col_bytes + val_bytes);
            if (col_bytes) tc::bulk_g2s(smem + P.off_col, p.col + (q0 - (q0 & 3)), col_bytes, cbar);
            if (val_bytes) tc::bulk_g2s(smem + P.off_val, p.val + (q0 - (q0 & 7)), val_bytes, cbar);
        }
        __syncwarp();
        tmem_alloc(s_taddr, kTmemCols);
    }

    // ---- dense warps: the first D units of the warp's code ring
    uint8_t* ring = smem + P.off_ring + (ctrl ? 0 : warp) * S * F::kSgBytes + lane * 16;
    int pj = wu0;  // next unit to request
    auto issue = [&](int stage) {
        if (pj < wu1) {
            const uint8_t* src = p.codes + (int64_t)pj * F::kSgBytes + lane * 16;
            uint8_t* dst = ring + stage * F::kSgBytes;
#pragma unroll
            for (int m = 0; m < V; ++m) tc::cp_async16(dst + m * 512, src + m * 512);
            ++pj;
        }
        tc::cp_async_commit();
    };
    if (!ctrl)
        for (int j = 0; j < D; ++j) issue(j);

    // ---- bookkeeping: contributors per tile, zeroed sparse sums, zero x past K
    for (int tl = tid; tl < ctiles; tl += kThreads) {
        const int ta_u = (t_first + tl) * nsg, tb_u = ta_u + nsg;
        int mask = 0;
        for (int v = 0; v < kVWarps; ++v)
            if (max(vbeg(v), ta_u) < min(vbeg(v + 1), tb_u)) mask |= 1 << v;
        s_tinfo[tl] = mask;
    }
    if (layer_csr)
        for (int i = tid; i < nrows * CM; i += kThreads) s_rowsum[i] = 0.f;
    {
        const int len = p.k_in, pad = nsg * kSgCols - len;
        for (int i = tid; i < B * pad; i += kThreads) {
            const int b = i / pad;
            xs[b * P.x_stride + len + (i - b * pad)] = 0;
        }
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t taddr = *s_taddr;
    const unsigned int ticket = *s_ticket;

    if (ctrl) {
        // ---- x may be written by the previous kernel of the stream: wait
        // for it (its lines were requested into L2 first: a hint only)
        {
            const int lines = (p.k_in * 2 + 127) / 128;
            for (int b = 0; b < B; ++b) {
                const char* xr = reinterpret_cast<const char*>(p.x + b * p.ldx);
                for (int l = lane; l < lines; l += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(xr + l * 128));
            }
        }
        tc::pdl_wait_previous();
        if (p.x_bulk) {
            if (lane == 0) {
                tc::mbar_expect_tx(xbar, (uint32_t)B * p.k_in * 2);
                for (int b = 0; b < B; ++b) tc::bulk_g2s(xs + b * P.x_stride, p.x + b * p.ldx, p.k_in * 2, xbar);
            }
        } else {
            for (int i = lane; i < B * p.k_in; i += 32) {
                const int b = i / p.k_in, k = i - b * p.k_in;
                xs[b * P.x_stride + k] = p.x[b * p.ldx + k];
            }
            tc::mbar_arrive(xbar);  // release: this lane's x stores before the phase completes
        }
    }

    // ---- sparse part (balanced): the CTA's entries [q0, q1) in kVThreads
    // equal shares; share t is summed per row (its first and last rows into
    // head/tail pieces, rows it holds whole straight into s_rowsum)
    const int q0 = __ldg(p.csr_cta + c), q1 = __ldg(p.csr_cta + c + 1);
    const int nz = q1 - q0;
    const bool has_csr = nz > 0;
    const int e_per = has_csr ? (nz + kVThreads - 1) / kVThreads : 1;
    const bool csr_in_smem = has_csr && nz <= P.csr_cap;
    const int* csr_col = csr_in_smem ? reinterpret_cast<const int*>(smem + P.off_col) + (q0 & 3) - q0 : p.col;
    const uint16_t* csr_val = csr_in_smem ? reinterpret_cast<const uint16_t*>(smem + P.off_val) + (q0 & 7) - q0 : p.val;
    auto share_begin = [&](int t) { return (int)min((int64_t)q1, (int64_t)q0 + (int64_t)t * e_per); };
    // row (relative to ra) of entry ca: the largest r with s_rp[r] <= ca (needs no x)
    auto share_row = [&](int ca) {
        int lo = 0, hi = nrows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_rp[mid] <= ca) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    auto sparse_share = [&](int t, int row0) {
        const int ca = share_begin(t);
        const int cb = (int)min((int64_t)q1, (int64_t)ca + e_per);
        if (ca >= cb) return;
        int cur = row0, nxt = s_rp[cur + 1];
        bool first = true;
        float acc[CM];
#pragma unroll
        for (int b = 0; b < CM; ++b) acc[b] = 0.f;
        auto emit = [&](bool last) {
            float* dstp;
            if (first) {
                s_headrow[t] = cur;
                dstp = s_head + t * CM;
            } else if (last) {
                s_tailrow[t] = cur;
                dstp = s_tail + t * CM;
            } else {
                dstp = s_rowsum + cur * CM;
            }
#pragma unroll
            for (int b = 0; b < CM; ++b) dstp[b] = acc[b];
        };
        for (int base = ca; base < cb; base += 8) {
            int cc[8];
            uint32_t vh[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int q = base + j;
                const bool in = q < cb;
                cc[j] = in ? csr_col[q] : 0;
                vh[j] = in ? (uint32_t)csr_val[q] : 0u;
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
                    if (SB || b < B) acc[b] = fmaf(v, h2f(xs[b * P.x_stride + cc[j]]), acc[b]);
            }
        }
        emit(true);
    };
    bool waits_ok = true;
    int srow[RG];  // starting row of each of this thread's shares (found before x arrives)
    if (!ctrl) {
        waits_ok = tc::mbar_wait(lbar, 0) && tc::mbar_wait(cbar, 0);
        if (has_csr)
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const int t = (warp * RG + r) * 32 + lane;
                s_headrow[t] = -1;
                s_tailrow[t] = -1;
                const int ca = share_begin(t);
                srow[r] = ca < q1 ? share_row(ca) : 0;
            }
    }

    // ---- dense warps
    if (!ctrl) {
        // this warp's TMEM: lanes of quarter warp % 4, columns (warp / 4) * 128 ...
        const uint32_t tw = taddr + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)((warp >> 2) * 128);
        TAB tg, tg8;
        auto load_tabs = [&](int tile) {
            const uint8_t* lt = luts + (tile - t_first) * kTileRows * F::kLutBytes;
            if constexpr (BITS == 3) {
                tg = tc::load_tab3(lt + g * F::kLutBytes);
                tg8 = tc::load_tab3(lt + (g + 8) * F::kLutBytes);
            } else {
                tg = tc::load_tab4(lt + g * F::kLutBytes);
                tg8 = tc::load_tab4(lt + (g + 8) * F::kLutBytes);
            }
        };
        auto read_stage = [&](int s, uint32_t (&w)[4 * V]) {
            const uint8_t* src = ring + s * F::kSgBytes;
#pragma unroll
            for (int m = 0; m < V; ++m) {
                const uint4 v = *reinterpret_cast<const uint4*>(src + m * 512);
                w[4 * m] = v.x, w[4 * m + 1] = v.y, w[4 * m + 2] = v.z, w[4 * m + 3] = v.w;
            }
        };
        auto x_arrived = [&]() -> bool {
            const bool t = lane == 0 ? mbar_test(xbar, 0) : false;
            return __shfl_sync(0xffffffffu, t, 0);
        };
        __syncwarp();

        // ---- ahead of x: decode the first units' quads into TMEM until x
        // is in shared memory (checked before every quad)
        int qp = 0;  // quads parked
        int s_read = 0, s_fill = D;
        // the SM's earlier CTAs of this kernel first (see g_pd_looped)
        if (nwu > 0) {
            bool go = false;
            for (int i = 0; i < kGatePolls && !go; ++i) {
                bool t = false;
                if (lane == 0) t = mbar_test(xbar, 0) || (int)(ld_relaxed(&g_pd_looped[smslot]) - ticket) >= 0;
                go = __shfl_sync(0xffffffffu, t, 0);
                if (!go) __nanosleep(256);
            }
        }
        if (nwu > 0) {
            const int pre = min(nwu, kPreUnits);
            int tab_tile = -1;
            bool stop = false;
            for (int u = 0; u < pre && !stop; ++u) {
                if (x_arrived()) break;
                tc::cp_async_wait<S - 2>();
                uint32_t w[4 * V];
                read_stage(s_read, w);
                const int tile = (wu0 + u) / nsg;
                if (tile != tab_tile) {
                    load_tabs(tile);
                    tab_tile = tile;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (q > 0 && x_arrived()) {
                        stop = true;
                        break;
                    }
                    uint32_t a[16];
                    decode_quad<BITS>(tg, tg8, w, q, a);
                    tmem_st16(tw + (uint32_t)(64 * u + 16 * q), a);
                    ++qp;
                }
                if (!stop) {  // the unit is parked whole: its stage is free
                    issue(s_fill);
                    s_read = s_read + 1 == S ? 0 : s_read + 1;
                    s_fill = s_fill + 1 == S ? 0 : s_fill + 1;
                }
            }
            tmem_wait_st();
        }
        if (!tc::mbar_wait(xbar, 0)) waits_ok = false;
        __syncwarp();

        // ---- every unit in order: the parked ones from TMEM (MMAs only),
        // a partly parked one quad by quad, the rest decoded
        const int xrow = g < B ? g : 0;  // batch column of this lane's B fragment (n = g)
        float d0[4], d1[4];
        int tile = wfirst, sg = wu0 - wfirst * nsg;
        int vw = warp * RG;                    // current virtual warp (the first non-empty one)
        int vend = vbeg(vw + 1) - wu0;         // its end (relative unit index)
        while (vend <= 0 && vw + 1 < (warp + 1) * RG) vend = vbeg(++vw + 1) - wu0;
        int vfirst = wfirst;                   // first tile of the current virtual warp
        auto zero_acc = [&]() {
#pragma unroll
            for (int q = 0; q < 4; ++q) d0[q] = d1[q] = 0.f;
        };
        // the current virtual warp's part of `tile`: the tile's sum when the
        // virtual warp holds it whole, else its slot (first or last tile it shares)
        auto flush_tile = [&]() {
            float rr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) rr[q] = d0[q] + d1[q];
            const int tl = tile - t_first;
            const int mask = s_tinfo[tl];
            float* dst = (mask & (mask - 1)) == 0 ? s_tsum + tl * TE
                                                  : s_slots + (vw * 2 + (tile == vfirst ? 0 : 1)) * TE;
            if constexpr (SB) {
                if (t4 == 0) {
                    dst[g] = rr[0];
                    dst[g + 8] = rr[2];
                }
            } else {
                const int col = 2 * t4;
                dst[g * CM + col] = rr[0];
                dst[g * CM + col + 1] = rr[1];
                dst[(g + 8) * CM + col] = rr[2];
                dst[(g + 8) * CM + col + 1] = rr[3];
            }
        };
        auto mma_quad = [&](const uint16_t* xb, int q, const uint32_t (&a)[16]) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xb + (4 * q + j) * 16);
                if (j & 1)
                    tc::mma16816(d1, a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3], xv.x, xv.y);
                else
                    tc::mma16816(d0, a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3], xv.x, xv.y);
            }
        };
        auto next_stage = [&](uint32_t (&w)[4 * V]) {
            tc::cp_async_wait<S - 2>();
            read_stage(s_read, w);
            issue(s_fill);
            s_read = s_read + 1 == S ? 0 : s_read + 1;
            s_fill = s_fill + 1 == S ? 0 : s_fill + 1;
        };
        const int nfull = qp >> 2, tq_part = qp & 3;
        // after a unit: the accumulators go to the tile's slot at the end of a
        // tile or of a virtual warp
        auto unit_done = [&](int u) {
            const bool tile_end = ++sg == nsg;
            const bool v_end = u + 1 == vend;
            if (tile_end || v_end) {
                flush_tile();
                __syncwarp();  // the tcgen05 loads that follow need the whole warp
                zero_acc();
                if (v_end && u + 1 < nwu) {  // the next virtual warp
                    ++vw;
                    vend = vbeg(vw + 1) - wu0;
                    vfirst = (wu0 + u + 1) / nsg;
                }
                if (tile_end && u + 1 < nwu) {
                    ++tile;
                    sg = 0;
                    load_tabs(tile);
                }
            }
        };
        if (nwu > 0) {
            load_tabs(tile);
            zero_acc();
        }
        int u = 0;
        // parked whole: MMAs only
#pragma unroll 1
        for (; u < nfull; ++u) {
            const uint16_t* xb = xs + xrow * P.x_stride + sg * kSgCols + 4 * t4;
            const uint32_t tcol = tw + (uint32_t)(64 * u);
            uint32_t a[16], b[16];
            tmem_ld16(tcol, a);
            tmem_ld16(tcol + 16, b);
            tmem_wait_ld(a, b);
            mma_quad(xb, 0, a);
            tmem_ld16(tcol + 32, a);
            mma_quad(xb, 1, b);
            tmem_wait_ld(a);
            tmem_ld16(tcol + 48, b);
            mma_quad(xb, 2, a);
            tmem_wait_ld(b);
            mma_quad(xb, 3, b);
            unit_done(u);
        }
        // parked in part: quad by quad
        if (tq_part > 0 && u < nwu) {
            const uint16_t* xb = xs + xrow * P.x_stride + sg * kSgCols + 4 * t4;
            const uint32_t tcol = tw + (uint32_t)(64 * u);
            uint32_t w[4 * V];
            next_stage(w);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t a[16];
                if (q < tq_part) {
                    tmem_ld16(tcol + 16 * q, a);
                    tmem_wait_ld(a);
                } else {
                    decode_quad<BITS>(tg, tg8, w, q, a);
                }
                mma_quad(xb, q, a);
            }
            unit_done(u);
            ++u;
        }
        // the sparse shares: the warps of the lower half before their decode
        // loop, the others after it, so that every sub-partition has a warp
        // decoding while another waits on the shares' loads
        const bool sparse_first = warp < (NW / 2);
        auto run_shares = [&]() {
            if (has_csr)
#pragma unroll
                for (int r = 0; r < RG; ++r) sparse_share((warp * RG + r) * 32 + lane, srow[r]);
            __syncwarp();
        };
        if (sparse_first) run_shares();
        // the rest: decoded here
#pragma unroll 1
        for (; u < nwu; ++u) {
            const uint16_t* xb = xs + xrow * P.x_stride + sg * kSgCols + 4 * t4;
            uint32_t w[4 * V];
            next_stage(w);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t a[16];
                decode_quad<BITS>(tg, tg8, w, q, a);
                mma_quad(xb, q, a);
            }
            unit_done(u);
        }
        if (!sparse_first) run_shares();
    }
    if (!waits_ok) atomicOr(p.status, tc::kStatusWaitTimeout);

    // ---- once every warp has left its loop: each output is the tile's sum
    // (or the virtual warps' parts of a shared tile, in order) plus the row's
    // sparse sum (interior sum, then the pieces of the shares that cut the
    // row: in share order, or by a warp for a long row); the control warp
    // frees TMEM (every tcgen05.ld has completed)
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    if (ctrl) tmem_dealloc(taddr, kTmemCols);
    if (tid == 0) atomicAdd(&g_pd_looped[smslot], 1u);  // this CTA's dense loops are done
    // rows cut into more than kLongPieces shares: their pieces are added into
    // the interior sum by a warp first (the loop below skips them)
    if (has_csr) {
        tc::add_long_rows<CM>(nrows, warp, kThreads / 32, lane, s_rp, q0, e_per, kVThreads, s_rowsum, s_headrow,
                              s_head, s_tailrow, s_tail);
        __syncthreads();
    }
    for (int idx = tid; idx < ctiles * TE; idx += kThreads) {
        const int tl = idx / TE, e = idx - tl * TE;
        const int row_l = e / CM, col = e - row_l * CM;
        const int tile = t_first + tl;
        const int row = tile * kTileRows + row_l;
        if (row >= p.n_out || col >= B) continue;
        const int mask = s_tinfo[tl];
        float sum = 0.f;
        if ((mask & (mask - 1)) == 0) {
            sum = s_tsum[idx];
        } else {
            for (int mm = mask; mm; mm &= mm - 1) {
                const int v = __ffs(mm) - 1;
                const int vfirst_v = vbeg(v) / nsg;
                sum += s_slots[(v * 2 + (tile == vfirst_v ? 0 : 1)) * TE + e];
            }
        }
        if (has_csr) {
            const int i = row - ra, rs = s_rp[i], re = s_rp[i + 1];
            if (re > rs) {
                float cs = s_rowsum[i * CM + col];
                const int tau_a = (rs - q0) / e_per, tau_b = min(kVThreads - 1, (re - 1 - q0) / e_per);
                for (int tau = tau_a; tau <= tau_b && tau_b - tau_a < tc::kLongPieces; ++tau) {
                    if (s_headrow[tau] == i) cs += s_head[tau * CM + col];
                    if (s_tailrow[tau] == i) cs += s_tail[tau * CM + col];
                }
                sum += cs;
            }
        }
        p.y[col * p.ldy + row] = f2h_rn(sum);
    }
}

}  // namespace pd
}  // namespace sqz
