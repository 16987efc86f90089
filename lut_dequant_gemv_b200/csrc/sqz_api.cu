// sqz_api.cu -- host side of the C ABI declared in include/sqz.h.
//
// Argument checks happen on the host before any CUDA call; device-content
// checks (CSR well-formedness) run in a validation kernel whose result the
// create call reads back.  Nothing here aborts, throws across the ABI or
// traps on the device.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <new>
#include <string>
#include <vector>

#include "../../include/sqz.h"
#include "kernels_basic.cuh"
#include "kernels_pd.cuh"
#include "kernels_tc.cuh"

namespace {

thread_local std::string g_last_error;

sqz_status fail(sqz_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

sqz_status cuda_fail(cudaError_t e, const char* what) {
    return fail(e == cudaErrorMemoryAllocation ? SQZ_ERR_OOM : SQZ_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorName(e), cudaGetErrorString(e));
}

#define SQZ_CUDA_TRY(expr, what)                 \
    do {                                         \
        cudaError_t e_ = (expr);                 \
        if (e_ != cudaSuccess) {                 \
            (void)cudaGetLastError();            \
            return cuda_fail(e_, what);          \
        }                                        \
    } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int sm_count_of_current_device() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

int max_smem_optin() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 232448;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || n <= 0)
        return 232448;
    return n;
}


}  // namespace

struct sqz_layer {
    int32_t n_out = 0, k_in = 0, bits = 0;
    int64_t nnz = 0;
    int64_t wpr = 0;  // 32-bit words per row of canonical codes
    int device = 0;
    int sm_count = 148;
    int smem_optin = 232448;
    int smem_budget = 232448;  // shared memory of one fused CTA (kCtasPerSm of them share an SM)
    int mac = SQZ_MAC_TENSOR_CORES;
    int csr_mode = SQZ_CSR_BALANCED;
    int predecode = 0;  // batches of 1..8: 1/8/16 take the kernel that decodes ahead of x into TMEM
    // The fused kernel serves every layer with N > 0 and K > 0 (columns past
    // K are padded inside the kernel-native layout).
    bool fused_ok = false;
    // canonical copies, kept only for layers whose batch-1 calls the fused
    // kernel cannot serve (the row-per-warp kernel reads them)
    uint32_t* codes = nullptr;
    uint16_t* lut = nullptr;
    bool canonical_released = false;
    // CSR copies, padded by 8 elements so that 16-byte aligned bulk copies
    // of any slice stay inside the allocation
    int32_t* rowptr = nullptr;
    int32_t* col = nullptr;
    uint16_t* val = nullptr;
    // kernel-native layout for the fused kernel
    int ntiles = 0, nsteps = 0, nsg = 0;
    int64_t units = 0;
    int grid = 0;                     // CTAs of a fused launch (one per SM)
    int32_t* csr_cta = nullptr;       // [grid + 1] (device): CSR entry range of each CTA's rows
    int32_t* cta_tiles = nullptr;     // [grid + 1] (device): first tile of each CTA, or nullptr (even split)
    int ctiles_max = 0;               // the most tiles one CTA owns
    uint8_t* codes_native = nullptr;  // [ntiles][nsg][sg_bytes]
    uint8_t* lut_native = nullptr;    // [ntiles*16][2 << bits] byte planes
    int* status = nullptr;            // [1]
    uint16_t* x_stage = nullptr;      // [SQZ_MAX_BATCH][k_in] for sqz_gemv_host
    uint16_t* y_stage = nullptr;      // [SQZ_MAX_BATCH][n_out]
    // sqz_gemv_host: copy-in, product and copy-out captured once per (host
    // buffers, shape, stream) and replayed as one graph launch
    struct HostGraph {
        const void* x;
        void* y;
        int32_t batch;
        int64_t ldx, ldy;
        cudaStream_t stream;
        cudaGraphExec_t exec;
        uint64_t used;
    };
    std::vector<HostGraph> host_graphs;
    uint64_t host_clock = 0;
    int64_t device_bytes = 0;
};

namespace {

void drop_host_graphs(sqz_layer* L) {
    for (auto& g : L->host_graphs) cudaGraphExecDestroy(g.exec);
    L->host_graphs.clear();
}

void free_layer(sqz_layer* L) {
    if (!L) return;
    drop_host_graphs(L);
    cudaFree(L->codes);
    cudaFree(L->lut);
    cudaFree(L->rowptr);
    cudaFree(L->col);
    cudaFree(L->val);
    cudaFree(L->codes_native);
    cudaFree(L->lut_native);
    cudaFree(L->status);
    cudaFree(L->csr_cta);
    cudaFree(L->cta_tiles);
    cudaFree(L->x_stage);
    cudaFree(L->y_stage);
    delete L;
}

template <class T>
sqz_status alloc(T** p, size_t count, sqz_layer* L, const char* what) {
    *p = nullptr;
    if (count == 0) return SQZ_OK;
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        *p = nullptr;
        return cuda_fail(e, what);
    }
    L->device_bytes += (int64_t)(count * sizeof(T));
    return SQZ_OK;
}

sqz_status check_desc(const sqz_layer_desc* d) {
    if (d->bits != 3 && d->bits != 4) return fail(SQZ_ERR_INVALID_ARG, "bits must be 3 or 4 (got %d)", d->bits);
    if (d->n_out < 0 || d->k_in < 0)
        return fail(SQZ_ERR_INVALID_ARG, "negative size (n_out=%d, k_in=%d)", d->n_out, d->k_in);
    const int kmult = d->bits == 3 ? 32 : 8;
    if (d->k_in % kmult != 0)
        return fail(SQZ_ERR_INVALID_ARG, "k_in=%d must be a multiple of %d for %d-bit codes (whole words per row)",
                    d->k_in, kmult, d->bits);
    if (d->nnz < 0 || d->nnz > INT32_MAX - 64) return fail(SQZ_ERR_INVALID_ARG, "nnz=%lld out of range", (long long)d->nnz);
    if ((int64_t)d->n_out * d->k_in > 0 && !d->codes) return fail(SQZ_ERR_INVALID_ARG, "codes is NULL");
    if (d->n_out > 0 && !d->lut) return fail(SQZ_ERR_INVALID_ARG, "lut is NULL");
    if (d->nnz > 0 && (!d->rowptr || !d->col || !d->val))
        return fail(SQZ_ERR_INVALID_ARG, "nnz=%lld but rowptr/col/val is NULL", (long long)d->nnz);
    if (d->nnz > 0 && d->k_in == 0) return fail(SQZ_ERR_INVALID_ARG, "nnz > 0 with k_in == 0");
    if (d->n_out >= INT32_MAX - 16) return fail(SQZ_ERR_INVALID_ARG, "n_out too large");
    return SQZ_OK;
}

sqz_status check_gemv_args(const sqz_layer* L, const void* x, int32_t batch, int64_t ldx, const void* y, int64_t ldy) {
    if (!L) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    if (batch < 1 || batch > SQZ_MAX_BATCH)
        return fail(SQZ_ERR_INVALID_ARG, "batch=%d outside [1, %d]", batch, SQZ_MAX_BATCH);
    if (ldx < L->k_in) return fail(SQZ_ERR_INVALID_ARG, "ldx=%lld < k_in=%d", (long long)ldx, L->k_in);
    if (ldy < L->n_out) return fail(SQZ_ERR_INVALID_ARG, "ldy=%lld < n_out=%d", (long long)ldy, L->n_out);
    if (L->k_in > 0 && !x) return fail(SQZ_ERR_INVALID_ARG, "x is NULL");
    if (L->n_out > 0 && !y) return fail(SQZ_ERR_INVALID_ARG, "y is NULL");
    return SQZ_OK;
}

// ------------------------------------------------------------ row per warp
template <int BITS, int B>
void launch_rowwarp(const sqz_layer* L, const uint16_t* x, int64_t ldx, uint16_t* y, int64_t ldy, cudaStream_t s) {
    const int64_t blocks = (L->n_out + 7) / 8;
    const unsigned grid = (unsigned)(blocks < 65535 * 8 ? blocks : 65535 * 8);
    sqz::gemv_rowwarp_kernel<BITS, B><<<grid, 256, 0, s>>>(L->codes, L->lut, L->rowptr, L->col, L->val, L->nnz, x,
                                                         ldx, y, ldy, L->n_out, L->k_in);
}

template <int BITS>
void dispatch_rowwarp(const sqz_layer* L, const uint16_t* x, int32_t batch, int64_t ldx, uint16_t* y, int64_t ldy,
                      cudaStream_t s) {
    switch (batch) {
#define SQZ_CASE(B) \
    case B: launch_rowwarp<BITS, B>(L, x, ldx, y, ldy, s); break;
        SQZ_CASE(1) SQZ_CASE(2) SQZ_CASE(3) SQZ_CASE(4) SQZ_CASE(5) SQZ_CASE(6) SQZ_CASE(7) SQZ_CASE(8)
        SQZ_CASE(9) SQZ_CASE(10) SQZ_CASE(11) SQZ_CASE(12) SQZ_CASE(13) SQZ_CASE(14) SQZ_CASE(15) SQZ_CASE(16)
#undef SQZ_CASE
        default: break;
    }
}

// ------------------------------------------------------------ fused kernel
template <int BITS, int NT, int MAC, bool SB, bool RW = false, int CM = (SB ? 1 : 8 * NT)>
sqz_status set_smem_attr(int bytes) {
    SQZ_CUDA_TRY(cudaFuncSetAttribute(sqz::tc::gemv_fused_kernel<BITS, NT, MAC, SB, RW, CM>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                 "cudaFuncSetAttribute");
    return SQZ_OK;
}

template <int BITS>
sqz_status prepare_fused_bits(int optin) {
    using namespace sqz::tc;
    sqz_status st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, true>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, false, 2>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, false, 4>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, false, 8>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 2, kMacTensor, false>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacCuda, true>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacMixed, true>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, true, true>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, true, 2>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, true, 4>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 1, kMacTensor, false, true, 8>(optin)) != SQZ_OK) return st;
    if ((st = set_smem_attr<BITS, 2, kMacTensor, false, true>(optin)) != SQZ_OK) return st;
    return SQZ_OK;
}

sqz_status prepare_fused_kernels(int optin) {
    sqz_status st = prepare_fused_bits<3>(optin);
    if (st != SQZ_OK) return st;
    if ((st = prepare_fused_bits<4>(optin)) != SQZ_OK) return st;
#define SQZ_PD_ATTR(BITS, SB, NW)                                                                            \
    SQZ_CUDA_TRY(cudaFuncSetAttribute(sqz::pd::gemv_pd_kernel<BITS, SB, NW>,                                 \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, optin),                   \
                 "cudaFuncSetAttribute")
    SQZ_PD_ATTR(3, true, 8);
    SQZ_PD_ATTR(3, false, 8);
    SQZ_PD_ATTR(4, true, 8);
    SQZ_PD_ATTR(4, false, 8);
    SQZ_PD_ATTR(3, true, 16);
    SQZ_PD_ATTR(3, false, 16);
    SQZ_PD_ATTR(4, true, 16);
    SQZ_PD_ATTR(4, false, 16);
#undef SQZ_PD_ATTR
    return SQZ_OK;
}

bool tc_grid_too_large(int n_out, int sm_count) { return sqz::tc::grid_size(n_out, sm_count) > sqz::tc::kMaxCtas; }

// The decode-ahead kernel's plan for a call, or false when it does not serve
// it (batch above 8, or x and the rings do not fit one CTA's shared memory).
// Two CTAs of 8 dense warps per SM when they fit in half an SM (`smem_half`),
// else one CTA of 16 dense warps; `force_nw` (8 or 16) asks for one shape.
bool pd_plan_for(int bits, int n_out, int k_in, int sm_count, int smem_half, int smem_optin, int batch, int force_nw,
                 sqz::pd::Plan* out, int* nw, int ctiles_max = 0) {
    if (batch < 1 || batch > 8 || n_out < 1 || k_in < 1) return false;
    if (tc_grid_too_large(n_out, sm_count)) return false;
    if (force_nw != 16) {
        const sqz::pd::Plan P = sqz::pd::make_plan(bits, n_out, k_in, batch, sm_count, smem_half, 8, ctiles_max);
        if (P.total <= smem_half) {
            *out = P;
            *nw = 8;
            return true;
        }
        if (force_nw == 8) return false;
    }
    const sqz::pd::Plan P = sqz::pd::make_plan(bits, n_out, k_in, batch, sm_count, smem_optin, 16, ctiles_max);
    if (P.total > smem_optin) return false;
    *out = P;
    *nw = 16;
    return true;
}

// Plan for a call, or false when the fused kernel cannot stage x.  A call
// first gets an SM's share (two CTAs per SM, so the next call's CTA can
// stream its weights while this one computes); one whose x does not fit
// there gets a whole SM; a batch whose x does not fit at all is staged in K
// chunks (several passes, fewest first).
// The device's side of a plan: SMs, the shared memory of one CTA when two
// share an SM, and the opt-in maximum of one CTA.
struct DeviceShape {
    int sm_count, smem_half, smem_optin;
};

bool plan_for(int bits, int n_out, int k_in, const DeviceShape& d, int batch, sqz::tc::Plan* out, int ctiles_max = 0) {
    const int nt = batch > 8 ? 2 : 1;
    const int grid = sqz::tc::grid_size(n_out, d.sm_count);
    const int nsg = ((k_in + 15) / 16 + sqz::tc::kSgSteps - 1) / sqz::tc::kSgSteps;
    for (int budget : {d.smem_half, d.smem_optin}) {
        sqz::tc::Plan P =
            sqz::tc::make_plan(bits, n_out, k_in, batch, nt, batch == 1, d.sm_count, budget, 1, ctiles_max);
        if (P.total <= budget && P.grid == grid) {
            *out = P;
            return true;
        }
    }
    if (batch > 1) {
        // fewest passes that still leave a ring of 4 stages per warp, else the
        // fewest passes that fit at all
        bool have = false;
        for (int passes = 2; passes <= nsg; ++passes) {
            sqz::tc::Plan P =
                sqz::tc::make_plan(bits, n_out, k_in, batch, nt, false, d.sm_count, d.smem_optin, passes, ctiles_max);
            if (P.passes != passes || P.total > d.smem_optin || P.grid != grid) continue;
            if (!have) {
                *out = P;
                have = true;
            }
            if (P.stages >= 4) {
                *out = P;
                return true;
            }
        }
        return have;
    }
    return false;
}

bool fused_plan(const sqz_layer* L, int batch, sqz::tc::Plan* out) {
    return plan_for(L->bits, L->n_out, L->k_in, DeviceShape{L->sm_count, L->smem_budget, L->smem_optin}, batch, out,
                    L->ctiles_max);
}

// Columns per launch and the plan of the first launch: the whole batch when
// a plan exists for it, else chunks of 8, 4, 2 or 1 columns (each launch
// reads the weights).  A batch above 8 whose x fits only in several passes
// runs as launches of 8 columns in one pass each when those fit: a pass
// gives each warp about one unit per tile, and the passes' barriers then
// cost more than decoding the weights twice.  Returns 0 when no fused plan
// exists (the row-per-warp kernel serves the call).
int launch_columns(int bits, int n_out, int k_in, const DeviceShape& d, int batch, sqz::tc::Plan* P,
                   int ctiles_max = 0) {
    int chunk = batch;
    bool fits = plan_for(bits, n_out, k_in, d, chunk, P, ctiles_max);
    if (fits && P->passes > 1) {
        // x staged in K chunks: the passes' barriers cost more than decoding
        // the weights again (from L2) in another launch once there are more
        // passes than launches -- take the widest single-pass column chunk
        // whose launches are fewer than the passes (measured on B200:
        // 5120x13824 at 8 columns, 55 us in 4 passes, 37 us as two launches
        // of 4).  Above 8 columns, launches of 8 whenever 8 fit one pass.
        for (int c : {8, 4, 2, 1}) {
            if (c >= batch) continue;
            sqz::tc::Plan Pc;
            if (!plan_for(bits, n_out, k_in, d, c, &Pc, ctiles_max) || Pc.passes != 1) continue;
            const int launches = (batch + c - 1) / c;
            if ((batch > 8 && c == 8) || launches < P->passes) {
                chunk = c;
                *P = Pc;
            }
            break;
        }
    }
    while (!fits && chunk > 1) {
        chunk = chunk > 8 ? 8 : chunk / 2;
        fits = plan_for(bits, n_out, k_in, d, chunk, P, ctiles_max);
    }
    return fits ? chunk : 0;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream is still running; it prefetches only
// weights before it waits for that kernel (griddepcontrol.wait).
template <int BITS, int NT, int MAC, bool SB, bool RW = false, int CM = (SB ? 1 : 8 * NT)>
cudaError_t launch_fused(const sqz::tc::Params& prm, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)prm.plan.grid);
    cfg.blockDim = dim3(sqz::tc::kThreads);
    cfg.dynamicSmemBytes = (size_t)prm.plan.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sqz::tc::gemv_fused_kernel<BITS, NT, MAC, SB, RW, CM>, prm);
}

// Batches 2..8 (one n-tile): the instantiation that carries the plan's
// number of batch columns (2, 4 or 8; the plan sized shared memory for it).
template <int BITS, bool RW>
cudaError_t launch_fused_one_tile(const sqz::tc::Params& prm, cudaStream_t s) {
    using namespace sqz::tc;
    switch (prm.plan.cm) {
        case 2: return launch_fused<BITS, 1, kMacTensor, false, RW, 2>(prm, s);
        case 4: return launch_fused<BITS, 1, kMacTensor, false, RW, 4>(prm, s);
        case 8: return launch_fused<BITS, 1, kMacTensor, false, RW, 8>(prm, s);
        default: return cudaErrorInvalidValue;
    }
}

// Batch 1 takes the requested multiply-accumulate unit; larger batches the
// tensor cores (one or two n-tiles of 8 batch columns).  The row-wise CSR
// comparison mode always uses the tensor cores.
template <int BITS>
cudaError_t launch_fused_bits(const sqz::tc::Params& prm, int batch, int mac, int csr_mode, cudaStream_t s) {
    using namespace sqz::tc;
    if (csr_mode == SQZ_CSR_ROWWISE) {
        if (batch > 8) return launch_fused<BITS, 2, kMacTensor, false, true>(prm, s);
        if (batch > 1) return launch_fused_one_tile<BITS, true>(prm, s);
        return launch_fused<BITS, 1, kMacTensor, true, true>(prm, s);
    }
    if (batch > 8) return launch_fused<BITS, 2, kMacTensor, false>(prm, s);
    if (batch > 1) return launch_fused_one_tile<BITS, false>(prm, s);
    if (mac == SQZ_MAC_CUDA_CORES) return launch_fused<BITS, 1, kMacCuda, true>(prm, s);
    if (mac == SQZ_MAC_MIXED) return launch_fused<BITS, 1, kMacMixed, true>(prm, s);
    return launch_fused<BITS, 1, kMacTensor, true>(prm, s);
}

template <int BITS, int NW>
cudaError_t launch_pd(const sqz::pd::Params& prm, bool single, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)prm.plan.grid);
    cfg.blockDim = dim3(sqz::pd::Shape<NW>::kThreads);
    cfg.dynamicSmemBytes = (size_t)prm.plan.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return single ? cudaLaunchKernelEx(&cfg, sqz::pd::gemv_pd_kernel<BITS, true, NW>, prm)
                  : cudaLaunchKernelEx(&cfg, sqz::pd::gemv_pd_kernel<BITS, false, NW>, prm);
}

// Whether a call takes the decode-ahead kernel: the handle's default options
// (tensor cores, balanced outliers), batch 1..8 and a plan that fits.
bool pd_serves(const sqz_layer* L, int32_t batch, sqz::pd::Plan* P, int* nw) {
    return L->fused_ok && L->predecode && L->mac == SQZ_MAC_TENSOR_CORES && L->csr_mode == SQZ_CSR_BALANCED &&
           pd_plan_for(L->bits, L->n_out, L->k_in, L->sm_count, L->smem_budget, L->smem_optin, batch,
                       L->predecode == 1 ? 0 : L->predecode, P, nw, L->ctiles_max) &&
           P->grid == L->grid;
}

sqz_status gemv_impl(const sqz_layer* L, const uint16_t* x, int32_t batch, int64_t ldx, uint16_t* y, int64_t ldy,
                     cudaStream_t s) {
    if (L->n_out == 0) return SQZ_OK;
    sqz::pd::Plan PP;
    int nw = 0;
    if (pd_serves(L, batch, &PP, &nw)) {
        sqz::pd::Params prm{};
        prm.codes = L->codes_native;
        prm.lutp = L->lut_native;
        prm.rowptr = L->rowptr;
        prm.col = L->col;
        prm.val = L->val;
        prm.x = x;
        prm.ldx = ldx;
        prm.y = y;
        prm.ldy = ldy;
        prm.status = L->status;
        prm.n_out = L->n_out;
        prm.k_in = L->k_in;
        prm.nsg = L->nsg;
        prm.ntiles = L->ntiles;
        prm.batch = batch;
        prm.has_csr = L->nnz > 0;
        prm.x_bulk = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (ldx % 8 == 0) && (L->k_in % 8 == 0);
        prm.plan = PP;
        prm.csr_cta = L->csr_cta;
        prm.cta_tiles = L->cta_tiles;
        const bool one = batch == 1;
        const cudaError_t e = L->bits == 3 ? (nw == 8 ? launch_pd<3, 8>(prm, one, s) : launch_pd<3, 16>(prm, one, s))
                                           : (nw == 8 ? launch_pd<4, 8>(prm, one, s) : launch_pd<4, 16>(prm, one, s));
        SQZ_CUDA_TRY(e, "fused gemv launch");
        return SQZ_OK;
    }
    sqz::tc::Plan P;
    const int chunk = L->fused_ok ? launch_columns(L->bits, L->n_out, L->k_in,
                                                   DeviceShape{L->sm_count, L->smem_budget, L->smem_optin}, batch, &P,
                                                   L->ctiles_max)
                                  : 0;
    const bool fits = chunk > 0;
    if (fits) {
        for (int b0 = 0; b0 < batch; b0 += chunk) {
            const int nb = batch - b0 < chunk ? batch - b0 : chunk;
            if (nb != chunk && !fused_plan(L, nb, &P)) return fail(SQZ_ERR_UNSUPPORTED, "no fused plan for %d columns", nb);
            const uint16_t* xc = x + (int64_t)b0 * ldx;
            sqz::tc::Params prm{};
            prm.codes = L->codes_native;
            prm.lutp = L->lut_native;
            prm.rowptr = L->rowptr;
            prm.col = L->col;
            prm.val = L->val;
            prm.x = xc;
            prm.ldx = ldx;
            prm.y = y + (int64_t)b0 * ldy;
            prm.ldy = ldy;
            prm.status = L->status;
            prm.n_out = L->n_out;
            prm.k_in = L->k_in;
            prm.nsg = L->nsg;
            prm.ntiles = L->ntiles;
            prm.batch = nb;
            prm.has_csr = L->nnz > 0;
            prm.x_bulk = (reinterpret_cast<uintptr_t>(xc) % 16 == 0) && (ldx % 8 == 0) && (L->k_in % 8 == 0);
            prm.plan = P;
            prm.csr_cta = L->csr_cta;
            prm.cta_tiles = L->cta_tiles;
            const cudaError_t e = L->bits == 3 ? launch_fused_bits<3>(prm, nb, L->mac, L->csr_mode, s)
                                               : launch_fused_bits<4>(prm, nb, L->mac, L->csr_mode, s);
            SQZ_CUDA_TRY(e, "fused gemv launch");
        }
    } else if (L->canonical_released) {
        return fail(SQZ_ERR_UNSUPPORTED, "no fused plan for this call and the canonical codes were released");
    } else if (L->bits == 3) {
        dispatch_rowwarp<3>(L, x, batch, ldx, y, ldy, s);
    } else {
        dispatch_rowwarp<4>(L, x, batch, ldx, y, ldy, s);
    }
    SQZ_CUDA_TRY(cudaGetLastError(), "gemv launch");
    return SQZ_OK;
}

// A split of the tiles over the CTAs by weight, for layers whose outliers
// are skewed: a CTA's time is its dense units (one per tile and 256-column
// super-group) plus its share of the sparse part, and a CTA whose rows hold
// many outliers should own fewer tiles.  Weight of a tile = its units x
// nnz_per_unit(bits) + its nonzeros (the nonzeros that cost about as much as
// one unit's decode, measured on B200: 100 at 3 bits; a 4-bit unit takes
// about 1.5x as long to decode, 150).  The CTAs take consecutive
// runs of at least one tile and at most twice the even split's count, split
// so that the heaviest run is as light as possible.  Used only when it
// lowers the heaviest CTA's weight by more than 5 %; otherwise (uniform
// outliers) the even split stays and `first` is left empty.
inline int64_t nnz_per_unit(int bits) { return bits == 3 ? 100 : 150; }
bool split_tiles_by_weight(const std::vector<int32_t>& rp, int n_out, int bits, int ntiles, int nsg, int grid,
                           std::vector<int32_t>* first, int* ctiles_max) {
    std::vector<int64_t> w((size_t)ntiles), pre((size_t)ntiles + 1, 0);
    for (int t = 0; t < ntiles; ++t) {
        const int r0 = t * sqz::tc::kTileRows, r1 = std::min(n_out, r0 + sqz::tc::kTileRows);
        w[t] = (int64_t)nsg * nnz_per_unit(bits) + (rp[r1] - rp[r0]);
        pre[t + 1] = pre[t] + w[t];
    }
    const int even_max = (ntiles + grid - 1) / grid, cap = 2 * even_max;
    auto heaviest = [&](const std::vector<int32_t>& f) {
        int64_t m = 0;
        for (int c = 0; c < grid; ++c) m = std::max(m, pre[f[c + 1]] - pre[f[c]]);
        return m;
    };
    std::vector<int32_t> even((size_t)grid + 1);
    for (int c = 0; c <= grid; ++c) even[c] = sqz::tc::tile_begin(ntiles, grid, c);
    // The split into `grid` runs of 1..cap consecutive tiles whose heaviest
    // run is lightest: the least bound W (binary search) for which runs packed
    // greedily up to W and `cap` tiles number at most `grid`; then, while there
    // are fewer runs than CTAs, the heaviest run of two or more tiles (the
    // first on ties) gives its last tile to a run of its own.
    auto pack = [&](int64_t W, std::vector<int32_t>* starts) {
        starts->clear();
        for (int t = 0; t < ntiles;) {
            if (w[t] > W) return false;
            starts->push_back(t);
            int64_t sum = 0;
            for (int k = 0; t < ntiles && k < cap && sum + w[t] <= W; ++k) sum += w[t++];
        }
        return (int)starts->size() <= grid;
    };
    std::vector<int32_t> split;
    int64_t lo = *std::max_element(w.begin(), w.end()), hi = pre[ntiles];
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (pack(mid, &split)) hi = mid;
        else lo = mid + 1;
    }
    if (!pack(lo, &split)) return false;
    split.push_back(ntiles);
    while ((int)split.size() - 1 < grid) {
        int best = -1;
        int64_t best_w = -1;
        for (int r = 0; r + 1 < (int)split.size(); ++r)
            if (split[r + 1] - split[r] >= 2 && pre[split[r + 1]] - pre[split[r]] > best_w) {
                best = r;
                best_w = pre[split[r + 1]] - pre[split[r]];
            }
        if (best < 0) return false;  // fewer tiles than CTAs: cannot happen (grid <= ntiles)
        split.insert(split.begin() + best + 1, split[best + 1] - 1);
    }
    int m = 0;
    for (int c = 0; c < grid; ++c) {
        const int n = split[c + 1] - split[c];
        if (n < 1 || n > cap) return false;  // the bounds could not all be met: keep the even split
        m = std::max(m, n);
    }
    if (!(heaviest(split) * 100 < heaviest(even) * 95)) return false;
    *first = split;
    *ctiles_max = m;
    return true;
}

// Kernel-native copies of codes and LUT and the fused kernel's status word.
sqz_status build_native(sqz_layer* L, cudaStream_t s) {
    using namespace sqz::tc;
    L->ntiles = (L->n_out + kTileRows - 1) / kTileRows;
    L->nsteps = (L->k_in + 15) / 16;
    L->nsg = (L->nsteps + kSgSteps - 1) / kSgSteps;
    L->grid = grid_size(L->n_out, L->sm_count);
    L->units = (int64_t)L->ntiles * L->nsg;
    const int sg_bytes = L->bits == 3 ? 1536 : 2048;
    const int lut_row = 2 << L->bits;
    sqz_status st;
    if ((st = alloc(&L->codes_native, (size_t)L->units * sg_bytes, L, "native codes")) != SQZ_OK) return st;
    if ((st = alloc(&L->lut_native, (size_t)L->ntiles * kTileRows * lut_row, L, "native lut")) != SQZ_OK) return st;
    if ((st = alloc(&L->status, 1, L, "status")) != SQZ_OK) return st;
    SQZ_CUDA_TRY(cudaMemsetAsync(L->status, 0, sizeof(int), s), "memset");
    if (L->units > 0) {
        const int64_t words = L->units * (sg_bytes / 4);
        int64_t blocks = (words + 255) / 256;
        if (blocks > (int64_t)L->sm_count * 16) blocks = (int64_t)L->sm_count * 16;
        if (L->bits == 3)
            repack_codes_kernel<3><<<(unsigned)blocks, 256, 0, s>>>(L->codes, L->lut, L->n_out, L->k_in, L->nsg, words,
                                                                    reinterpret_cast<uint32_t*>(L->codes_native));
        else
            repack_codes_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(L->codes, L->lut, L->n_out, L->k_in, L->nsg, words,
                                                                    reinterpret_cast<uint32_t*>(L->codes_native));
        SQZ_CUDA_TRY(cudaGetLastError(), "repack codes");
    }
    if (L->ntiles > 0) {
        const int rows = L->ntiles * kTileRows;
        const int blocks = (rows + 255) / 256;
        if (L->bits == 3)
            sqz::tc::repack_lut_kernel<3><<<blocks, 256, 0, s>>>(L->lut, L->n_out, rows, L->lut_native);
        else
            sqz::tc::repack_lut_kernel<4><<<blocks, 256, 0, s>>>(L->lut, L->n_out, rows, L->lut_native);
        SQZ_CUDA_TRY(cudaGetLastError(), "repack lut");
    }
    // Tiles of every CTA: the even split, or -- when the outliers are skewed
    // enough -- a split by weight (see split_tiles_by_weight)
    L->ctiles_max = (L->ntiles + L->grid - 1) / L->grid;
    if (L->nnz > 0 && L->grid > 1) {
        std::vector<int32_t> rp((size_t)L->n_out + 1), first;
        SQZ_CUDA_TRY(cudaMemcpyAsync(rp.data(), L->rowptr, rp.size() * 4, cudaMemcpyDeviceToHost, s), "rowptr read");
        SQZ_CUDA_TRY(cudaStreamSynchronize(s), "rowptr read");
        if (split_tiles_by_weight(rp, L->n_out, L->bits, L->ntiles, L->nsg, L->grid, &first, &L->ctiles_max)) {
            if ((st = alloc(&L->cta_tiles, (size_t)L->grid + 1, L, "CTA tiles")) != SQZ_OK) return st;
            SQZ_CUDA_TRY(cudaMemcpyAsync(L->cta_tiles, first.data(), first.size() * 4, cudaMemcpyHostToDevice, s),
                         "CTA tiles copy");
            SQZ_CUDA_TRY(cudaStreamSynchronize(s), "CTA tiles copy");  // `first` is a host temporary
        }
    }
    // CSR entry range of every CTA's rows (device array read by each launch)
    if ((st = alloc(&L->csr_cta, (size_t)L->grid + 1, L, "CTA bounds")) != SQZ_OK) return st;
    if (L->nnz > 0) {
        if (L->grid > kMaxCtas) return fail(SQZ_ERR_UNSUPPORTED, "%d CTAs exceed the fused kernel's %d", L->grid, kMaxCtas);
        csr_cta_bounds_kernel<<<(L->grid + 256) / 256, 256, 0, s>>>(L->rowptr, L->cta_tiles, L->n_out, L->ntiles,
                                                                    L->grid, L->csr_cta);
        SQZ_CUDA_TRY(cudaGetLastError(), "CTA bounds");
    } else {
        SQZ_CUDA_TRY(cudaMemsetAsync(L->csr_cta, 0, sizeof(int32_t) * ((size_t)L->grid + 1), s), "memset");
    }
    return SQZ_OK;
}

}  // namespace

extern "C" {

sqz_status sqz_create_layer(const sqz_layer_desc* desc, void* stream, sqz_layer_t* out) {
    if (out) *out = nullptr;
    if (!desc || !out) return fail(SQZ_ERR_INVALID_ARG, "desc and out must be non-NULL");
    sqz_status st = check_desc(desc);
    if (st != SQZ_OK) return st;
    cudaStream_t s = as_stream(stream);

    sqz_layer* L = new (std::nothrow) sqz_layer();
    if (!L) return fail(SQZ_ERR_OOM, "host allocation of the layer handle failed");
    L->n_out = desc->n_out;
    L->k_in = desc->k_in;
    L->bits = desc->bits;
    L->nnz = desc->nnz;
    L->wpr = (int64_t)desc->k_in * desc->bits / 32;
    L->sm_count = sm_count_of_current_device();
    L->smem_optin = max_smem_optin();
    {
        // an SM's shared memory split between kCtasPerSm CTAs, less the 1 KiB
        // the hardware reserves per CTA
        int dev = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
            per_sm = 233472;
        const int share = per_sm / sqz::tc::kCtasPerSm - 1024;
        L->smem_budget = share < L->smem_optin ? share : L->smem_optin;
    }
    cudaGetDevice(&L->device);

    const size_t n = (size_t)desc->n_out, lut_n = n << desc->bits, code_n = n * (size_t)L->wpr;
    const size_t nnz = (size_t)desc->nnz;
#define SQZ_STEP(expr)                 \
    do {                               \
        sqz_status s_ = (expr);        \
        if (s_ != SQZ_OK) {            \
            free_layer(L);             \
            return s_;                 \
        }                              \
    } while (0)
#define SQZ_CUDA_STEP(expr, what)               \
    do {                                        \
        cudaError_t e_ = (expr);                \
        if (e_ != cudaSuccess) {                \
            (void)cudaGetLastError();           \
            free_layer(L);                      \
            return cuda_fail(e_, what);         \
        }                                       \
    } while (0)

    SQZ_STEP(prepare_fused_kernels(L->smem_optin));
    SQZ_STEP(alloc(&L->codes, code_n, L, "codes allocation"));
    SQZ_STEP(alloc(&L->lut, lut_n, L, "lut allocation"));
    if (nnz > 0) {
        SQZ_STEP(alloc(&L->rowptr, n + 1 + 8, L, "rowptr allocation"));
        SQZ_STEP(alloc(&L->col, nnz + 8, L, "col allocation"));
        SQZ_STEP(alloc(&L->val, nnz + 8, L, "val allocation"));
    }
    SQZ_STEP(alloc(&L->x_stage, (size_t)SQZ_MAX_BATCH * desc->k_in, L, "x staging allocation"));
    SQZ_STEP(alloc(&L->y_stage, (size_t)SQZ_MAX_BATCH * n, L, "y staging allocation"));

    if (code_n)
        SQZ_CUDA_STEP(cudaMemcpyAsync(L->codes, desc->codes, code_n * 4, cudaMemcpyDeviceToDevice, s), "codes copy");
    if (lut_n)
        SQZ_CUDA_STEP(cudaMemcpyAsync(L->lut, desc->lut, lut_n * 2, cudaMemcpyDeviceToDevice, s), "lut copy");
    if (nnz > 0) {
        SQZ_CUDA_STEP(cudaMemsetAsync(L->rowptr, 0, (n + 1 + 8) * 4, s), "rowptr clear");
        SQZ_CUDA_STEP(cudaMemsetAsync(L->col, 0, (nnz + 8) * 4, s), "col clear");
        SQZ_CUDA_STEP(cudaMemsetAsync(L->val, 0, (nnz + 8) * 2, s), "val clear");
        SQZ_CUDA_STEP(cudaMemcpyAsync(L->rowptr, desc->rowptr, (n + 1) * 4, cudaMemcpyDeviceToDevice, s), "rowptr copy");
        SQZ_CUDA_STEP(cudaMemcpyAsync(L->col, desc->col, nnz * 4, cudaMemcpyDeviceToDevice, s), "col copy");
        SQZ_CUDA_STEP(cudaMemcpyAsync(L->val, desc->val, nnz * 2, cudaMemcpyDeviceToDevice, s), "val copy");

        int* d_flag = nullptr;
        SQZ_CUDA_STEP(cudaMalloc(&d_flag, sizeof(int)), "validation flag allocation");
        int h_flag = 0;
        cudaError_t e = cudaMemsetAsync(d_flag, 0, sizeof(int), s);
        if (e == cudaSuccess) {
            const int64_t work = (nnz > n + 1 ? (int64_t)nnz : (int64_t)n + 1);
            int64_t blocks = (work + 255) / 256;
            if (blocks > (int64_t)L->sm_count * 8) blocks = (int64_t)L->sm_count * 8;
            sqz::validate_csr_kernel<<<(unsigned)blocks, 256, 0, s>>>(L->rowptr, L->col, L->n_out, L->k_in, L->nnz,
                                                                        d_flag);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaMemcpyAsync(&h_flag, d_flag, sizeof(int), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        cudaFree(d_flag);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            free_layer(L);
            return cuda_fail(e, "CSR validation");
        }
        if (h_flag) {
            free_layer(L);
            return fail(SQZ_ERR_INVALID_ARG, "malformed CSR:%s%s%s%s", (h_flag & 1) ? " rowptr[0]!=0" : "",
                        (h_flag & 2) ? " rowptr[N]!=nnz" : "", (h_flag & 4) ? " rowptr decreasing" : "",
                        (h_flag & 8) ? " column outside [0,K)" : "");
        }
    }
    L->fused_ok = L->n_out > 0 && L->k_in > 0 && sqz::tc::grid_size(L->n_out, L->sm_count) <= sqz::tc::kMaxCtas;
    if (L->fused_ok) SQZ_STEP(build_native(L, s));
    SQZ_CUDA_STEP(cudaStreamSynchronize(s), "layer creation");
    // When the fused kernel serves one batch column, it serves every batch
    // (larger batches fall back to launches of fewer columns, down to one),
    // so the canonical codes and LUT -- read only by the row-per-warp kernel
    // -- are dropped: the handle then holds the compressed weights once.
    sqz::tc::Plan plan1;
    if (L->fused_ok && fused_plan(L, 1, &plan1)) {
        cudaFree(L->codes);
        cudaFree(L->lut);
        L->device_bytes -= (int64_t)(code_n * 4 + lut_n * 2);
        L->codes = nullptr;
        L->lut = nullptr;
        L->canonical_released = true;
    }
#undef SQZ_STEP
#undef SQZ_CUDA_STEP
    *out = L;
    return SQZ_OK;
}

sqz_status sqz_gemv(sqz_layer_t layer, const uint16_t* x, int32_t batch, int64_t ldx, uint16_t* y, int64_t ldy,
                    void* stream) {
    sqz_status st = check_gemv_args(layer, x, batch, ldx, y, ldy);
    if (st != SQZ_OK) return st;
    return gemv_impl(layer, x, batch, ldx, y, ldy, as_stream(stream));
}

}  // extern "C"

namespace {

// Device addresses of page-locked host buffers (nullptr: pageable memory).
struct HostMaps {
    bool x_pinned = false;
    uint16_t* y = nullptr;
};
HostMaps host_maps(const uint16_t* x_host, uint16_t* y_host) {
    HostMaps m;
    cudaPointerAttributes a{};
    m.x_pinned = cudaPointerGetAttributes(&a, x_host) == cudaSuccess && a.type == cudaMemoryTypeHost;
    a = cudaPointerAttributes{};
    if (cudaPointerGetAttributes(&a, y_host) == cudaSuccess && a.type == cudaMemoryTypeHost && a.devicePointer)
        m.y = static_cast<uint16_t*>(a.devicePointer);
    (void)cudaGetLastError();
    return m;
}

// Bring x in, run the product, take y out, all on stream s.  x goes to the
// handle's staging buffer by a copy-engine transfer.  A page-locked y is
// written by the product kernel's own stores through its device mapping (a
// copy-engine transfer after the kernel took 2-4 us longer per call); a
// pageable y goes through the staging buffer and a copy back.
sqz_status enqueue_host_call(const sqz_layer* L, const uint16_t* x_host, int32_t batch, int64_t ldx, uint16_t* y_host,
                             int64_t ldy, cudaStream_t s, const HostMaps& m) {
    sqz_status st;
    if (L->k_in > 0) {
        const size_t row = (size_t)L->k_in * 2;
        const cudaError_t e = (ldx == L->k_in || batch == 1)
                                  ? cudaMemcpyAsync(L->x_stage, x_host, row * batch, cudaMemcpyHostToDevice, s)
                                  : cudaMemcpy2DAsync(L->x_stage, row, x_host, (size_t)ldx * 2, row, (size_t)batch,
                                                      cudaMemcpyHostToDevice, s);
        SQZ_CUDA_TRY(e, "x host-to-device copy");
    }
    if (m.y) return gemv_impl(L, L->x_stage, batch, L->k_in, m.y, ldy, s);
    st = gemv_impl(L, L->x_stage, batch, L->k_in, L->y_stage, L->n_out, s);
    if (st != SQZ_OK) return st;
    if (L->n_out > 0) {
        const size_t row = (size_t)L->n_out * 2;
        const cudaError_t e = (ldy == L->n_out || batch == 1)
                                  ? cudaMemcpyAsync(y_host, L->y_stage, row * batch, cudaMemcpyDeviceToHost, s)
                                  : cudaMemcpy2DAsync(y_host, (size_t)ldy * 2, L->y_stage, row, row, (size_t)batch,
                                                      cudaMemcpyDeviceToHost, s);
        SQZ_CUDA_TRY(e, "y device-to-host copy");
    }
    return SQZ_OK;
}

constexpr size_t kHostGraphsPerLayer = 64;

// The cached graph of this call, captured on first use; nullptr when the
// call cannot be captured (the legacy default stream, or a stream that is
// already being captured), in which case the caller enqueues it directly.
cudaGraphExec_t host_graph(sqz_layer* L, const uint16_t* x_host, int32_t batch, int64_t ldx, uint16_t* y_host,
                           int64_t ldy, cudaStream_t s, const HostMaps& m) {
    if (s == nullptr || s == cudaStreamLegacy || s == cudaStreamPerThread) return nullptr;
    if (!m.x_pinned || !m.y) return nullptr;  // pageable memory: copied directly, not captured
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
    for (auto& g : L->host_graphs)
        if (g.x == x_host && g.y == y_host && g.batch == batch && g.ldx == ldx && g.ldy == ldy && g.stream == s) {
            g.used = ++L->host_clock;
            return g.exec;
        }
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    const sqz_status st = enqueue_host_call(L, x_host, batch, ldx, y_host, ldy, s, m);
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(s, &graph);
    cudaGraphExec_t exec = nullptr;
    if (st == SQZ_OK && e == cudaSuccess && graph && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) exec = nullptr;
    if (graph) cudaGraphDestroy(graph);
    (void)cudaGetLastError();
    if (!exec) return nullptr;
    if (L->host_graphs.size() >= kHostGraphsPerLayer) {  // drop the least recently used
        size_t old = 0;
        for (size_t i = 1; i < L->host_graphs.size(); ++i)
            if (L->host_graphs[i].used < L->host_graphs[old].used) old = i;
        cudaGraphExecDestroy(L->host_graphs[old].exec);
        L->host_graphs.erase(L->host_graphs.begin() + (ptrdiff_t)old);
    }
    L->host_graphs.push_back({x_host, y_host, batch, ldx, ldy, s, exec, ++L->host_clock});
    return exec;
}

}  // namespace

extern "C" {

sqz_status sqz_gemv_host(sqz_layer_t layer, const uint16_t* x_host, int32_t batch, int64_t ldx, uint16_t* y_host,
                         int64_t ldy, void* stream) {
    sqz_status st = check_gemv_args(layer, x_host, batch, ldx, y_host, ldy);
    if (st != SQZ_OK) return st;
    cudaStream_t s = as_stream(stream);
    const HostMaps m = host_maps(x_host, y_host);
    if (cudaGraphExec_t exec = host_graph(layer, x_host, batch, ldx, y_host, ldy, s, m)) {
        SQZ_CUDA_TRY(cudaGraphLaunch(exec, s), "graph launch");
    } else if ((st = enqueue_host_call(layer, x_host, batch, ldx, y_host, ldy, s, m)) != SQZ_OK) {
        return st;
    }
    SQZ_CUDA_TRY(cudaStreamSynchronize(s), "stream synchronize");
    return SQZ_OK;
}

sqz_status sqz_plan_query(int32_t n_out, int32_t k_in, int32_t bits, int32_t batch, int32_t sm_count,
                          int32_t smem_per_sm, int32_t smem_optin, int32_t predecode, sqz_plan_info* out) {
    if (!out) return fail(SQZ_ERR_INVALID_ARG, "out is NULL");
    *out = sqz_plan_info{};
    if (bits != 3 && bits != 4) return fail(SQZ_ERR_INVALID_ARG, "bits must be 3 or 4 (got %d)", bits);
    if (n_out < 1 || k_in < 1) return fail(SQZ_ERR_INVALID_ARG, "n_out and k_in must be positive");
    if (batch < 1 || batch > SQZ_MAX_BATCH) return fail(SQZ_ERR_INVALID_ARG, "batch must lie in [1, %d]", SQZ_MAX_BATCH);
    if (sm_count < 1 || smem_per_sm < 1 || smem_optin < 1)
        return fail(SQZ_ERR_INVALID_ARG, "sm_count, smem_per_sm and smem_optin must be positive");
    const int share = smem_per_sm / sqz::tc::kCtasPerSm - 1024;
    const DeviceShape d{sm_count, share < smem_optin ? share : smem_optin, smem_optin};
    const int grid = sqz::tc::grid_size(n_out, sm_count);
    sqz::pd::Plan PP;
    int nw = 0;
    if (predecode != 0 && predecode != 1 && predecode != 8 && predecode != 16)
        return fail(SQZ_ERR_INVALID_ARG, "predecode must be 0, 1, 8 or 16 (got %d)", predecode);
    if (predecode &&
        pd_plan_for(bits, n_out, k_in, sm_count, d.smem_half, smem_optin, batch, predecode == 1 ? 0 : predecode, &PP,
                    &nw)) {
        out->fused = 1;
        out->predecode = 1;
        out->columns_per_launch = batch;
        out->launches = 1;
        out->grid = PP.grid;
        out->threads = (nw + 1) * 32;
        out->smem_bytes = PP.total;
        out->ctas_per_sm = nw == 8 ? 2 : 1;
        out->passes = 1;
        out->ring_stages = sqz::pd::kStages;
        out->csr_stage_entries = PP.csr_cap;
        return SQZ_OK;
    }
    sqz::tc::Plan P{};
    const int chunk = grid <= sqz::tc::kMaxCtas ? launch_columns(bits, n_out, k_in, d, batch, &P) : 0;
    if (chunk == 0) return SQZ_OK;  // fused = 0: the row-per-warp kernel
    out->fused = 1;
    out->columns_per_launch = chunk;
    out->launches = (batch + chunk - 1) / chunk;
    out->grid = P.grid;
    out->threads = sqz::tc::kThreads;
    out->smem_bytes = P.total;
    out->ctas_per_sm = P.total <= d.smem_half ? sqz::tc::kCtasPerSm : 1;
    out->passes = P.passes;
    out->ring_stages = P.stages;
    out->csr_stage_entries = P.csr_cap;
    return SQZ_OK;
}

sqz_status sqz_tile_split_query(const int32_t* rowptr, int32_t n_out, int32_t k_in, int32_t bits, int32_t sm_count,
                                int32_t* first, int32_t* weighted) {
    if (!rowptr || !first || !weighted) return fail(SQZ_ERR_INVALID_ARG, "rowptr, first and weighted must not be NULL");
    *weighted = 0;
    if (bits != 3 && bits != 4) return fail(SQZ_ERR_INVALID_ARG, "bits must be 3 or 4 (got %d)", bits);
    if (n_out < 1 || k_in < 1) return fail(SQZ_ERR_INVALID_ARG, "n_out and k_in must be positive");
    if (sm_count < 1) return fail(SQZ_ERR_INVALID_ARG, "sm_count must be positive");
    if (rowptr[0] != 0) return fail(SQZ_ERR_INVALID_ARG, "rowptr[0] must be 0");
    for (int32_t i = 0; i < n_out; ++i)
        if (rowptr[i + 1] < rowptr[i]) return fail(SQZ_ERR_INVALID_ARG, "rowptr decreases at row %d", i);
    using namespace sqz::tc;
    const int ntiles = (n_out + kTileRows - 1) / kTileRows;
    const int grid = grid_size(n_out, sm_count);
    const int nsg = ((k_in + 15) / 16 + kSgSteps - 1) / kSgSteps;
    std::vector<int32_t> rp(rowptr, rowptr + (size_t)n_out + 1), split;
    int ctiles_max = 0;
    // the same condition and function as layer creation
    if (rp[(size_t)n_out] > 0 && grid > 1 && split_tiles_by_weight(rp, n_out, bits, ntiles, nsg, grid, &split, &ctiles_max)) {
        std::copy(split.begin(), split.end(), first);
        *weighted = 1;
    } else {
        for (int c = 0; c <= grid; ++c) first[c] = tile_begin(ntiles, grid, c);
    }
    return SQZ_OK;
}

sqz_status sqz_debug_dequant(sqz_layer_t layer, uint16_t* w_out, void* stream) {
    if (!layer) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    const sqz_layer* L = layer;
    if ((int64_t)L->n_out * L->k_in == 0) return SQZ_OK;
    if (!w_out) return fail(SQZ_ERR_INVALID_ARG, "w_out is NULL");
    cudaStream_t s = as_stream(stream);
    const int grid = L->sm_count * 4;
    if (!L->fused_ok) {
        if (L->bits == 3)
            sqz::dequant_canonical_kernel<3><<<grid, 256, 0, s>>>(L->codes, L->lut, L->n_out, L->k_in, w_out);
        else
            sqz::dequant_canonical_kernel<4><<<grid, 256, 0, s>>>(L->codes, L->lut, L->n_out, L->k_in, w_out);
    } else if (L->bits == 3)
        sqz::tc::dequant_native_kernel<3><<<grid, 256, 0, s>>>(L->codes_native, L->lut_native, L->n_out, L->k_in,
                                                               L->nsg, L->units, w_out);
    else
        sqz::tc::dequant_native_kernel<4><<<grid, 256, 0, s>>>(L->codes_native, L->lut_native, L->n_out, L->k_in,
                                                               L->nsg, L->units, w_out);
    SQZ_CUDA_TRY(cudaGetLastError(), "dequant launch");
    return SQZ_OK;
}

sqz_status sqz_layer_info(sqz_layer_t layer, int32_t* n_out, int32_t* k_in, int32_t* bits, int64_t* nnz,
                          int64_t* device_bytes) {
    if (!layer) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    if (n_out) *n_out = layer->n_out;
    if (k_in) *k_in = layer->k_in;
    if (bits) *bits = layer->bits;
    if (nnz) *nnz = layer->nnz;
    if (device_bytes) *device_bytes = layer->device_bytes;
    return SQZ_OK;
}

sqz_status sqz_layer_set_mac(sqz_layer_t layer, int32_t mac) {
    if (!layer) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    if (mac != SQZ_MAC_TENSOR_CORES && mac != SQZ_MAC_CUDA_CORES && mac != SQZ_MAC_MIXED)
        return fail(SQZ_ERR_INVALID_ARG, "unknown MAC unit %d", mac);
    layer->mac = mac;
    drop_host_graphs(layer);  // captured launches used the previous kernel
    return SQZ_OK;
}

sqz_status sqz_layer_set_csr_mode(sqz_layer_t layer, int32_t mode) {
    if (!layer) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    if (mode != SQZ_CSR_BALANCED && mode != SQZ_CSR_ROWWISE) return fail(SQZ_ERR_INVALID_ARG, "unknown CSR mode %d", mode);
    layer->csr_mode = mode;
    drop_host_graphs(layer);
    return SQZ_OK;
}

sqz_status sqz_layer_set_predecode(sqz_layer_t layer, int32_t enable) {
    if (!layer) return fail(SQZ_ERR_INVALID_ARG, "layer is NULL");
    if (enable != 0 && enable != 1 && enable != 8 && enable != 16)
        return fail(SQZ_ERR_INVALID_ARG, "enable must be 0, 1, 8 or 16 (got %d)", enable);
    layer->predecode = enable;
    drop_host_graphs(layer);
    return SQZ_OK;
}

sqz_status sqz_layer_status(sqz_layer_t layer, void* stream, int32_t* status) {
    if (!layer || !status) return fail(SQZ_ERR_INVALID_ARG, "layer and status must be non-NULL");
    *status = 0;
    if (!layer->status) return SQZ_OK;
    cudaStream_t s = as_stream(stream);
    int h = 0;
    SQZ_CUDA_TRY(cudaMemcpyAsync(&h, layer->status, sizeof(int), cudaMemcpyDeviceToHost, s), "status read");
    SQZ_CUDA_TRY(cudaMemsetAsync(layer->status, 0, sizeof(int), s), "status clear");
    SQZ_CUDA_TRY(cudaStreamSynchronize(s), "stream synchronize");
    *status = h;
    if (h & sqz::tc::kStatusWaitTimeout)
        return fail(SQZ_ERR_TIMEOUT, "a bounded device wait gave up (status 0x%x): y of the affected call is undefined",
                    h);
    return SQZ_OK;
}

sqz_status sqz_destroy(sqz_layer_t layer) {
    free_layer(layer);
    return SQZ_OK;
}

sqz_status sqz_fp16_gemv(const uint16_t* w, int32_t n_out, int32_t k_in, int64_t ldw, const uint16_t* x,
                         int32_t batch, int64_t ldx, uint16_t* y, int64_t ldy, void* stream) {
    if (n_out < 0 || k_in < 0) return fail(SQZ_ERR_INVALID_ARG, "negative size");
    if (batch < 1 || batch > SQZ_MAX_BATCH)
        return fail(SQZ_ERR_INVALID_ARG, "batch=%d outside [1, %d]", batch, SQZ_MAX_BATCH);
    if (ldw < k_in || ldx < k_in || ldy < n_out) return fail(SQZ_ERR_INVALID_ARG, "leading dimension too small");
    if ((int64_t)n_out * k_in > 0 && (!w || !x)) return fail(SQZ_ERR_INVALID_ARG, "w or x is NULL");
    if (n_out > 0 && !y) return fail(SQZ_ERR_INVALID_ARG, "y is NULL");
    if (n_out == 0) return SQZ_OK;
    cudaStream_t s = as_stream(stream);
    const int vec_ok = ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(x)) % 16 == 0) &&
                       ldw % 8 == 0 && ldx % 8 == 0 && k_in % 8 == 0;
    const int64_t blocks = (n_out + 7) / 8;
    const unsigned grid = (unsigned)(blocks < 65535 * 8 ? blocks : 65535 * 8);
    switch (batch) {
#define SQZ_CASE(B) \
    case B: sqz::fp16_gemv_kernel<B><<<grid, 256, 0, s>>>(w, ldw, x, ldx, y, ldy, n_out, k_in, vec_ok); break;
        SQZ_CASE(1) SQZ_CASE(2) SQZ_CASE(3) SQZ_CASE(4) SQZ_CASE(5) SQZ_CASE(6) SQZ_CASE(7) SQZ_CASE(8)
        SQZ_CASE(9) SQZ_CASE(10) SQZ_CASE(11) SQZ_CASE(12) SQZ_CASE(13) SQZ_CASE(14) SQZ_CASE(15) SQZ_CASE(16)
#undef SQZ_CASE
        default: break;
    }
    SQZ_CUDA_TRY(cudaGetLastError(), "fp16 gemv launch");
    return SQZ_OK;
}

const char* sqz_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

// Lets other translation units of the library report a message through
// sqz_last_error(); not exported.
void sqz_internal_set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

extern "C" {

int32_t sqz_version(void) { return 300; }

}  // extern "C"
