// sqz_noalloc.cu -- CSR well-formedness check that allocates no device memory.
//
// sqz_create_layer validates an outlier matrix with a kernel that reports
// into a flag word it cudaMalloc's for the occasion.  Some callers cannot
// allocate device memory at the point where they want that check: serving
// loops that must never take the implicit device synchronisation of
// cudaMalloc/cudaFree, and runtimes that reserve all of their device memory
// up front and forbid allocations afterwards.  For them sqz_check_csr_static
// runs the same validation kernel with its flag word in a fixed, file-scope
// device array instead.  It reads the verdict back and synchronises its
// stream, so it cannot run inside a CUDA-graph capture: it refuses a stream
// that is being captured.
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/sqz.h"
#include "kernels_basic.cuh"

void sqz_internal_set_last_error(const char* msg);

namespace {

// Scratch of sqz_check_csr_static: 64 int32 words (256 bytes) on every GPU
// that loads the library, held until the process exits.  Word 0 receives
// the validation flags; the check uses no other word, whatever the size of
// the matrix it checks.
constexpr int kCheckScratchWords = 64;
__device__ __align__(256) int g_check_scratch[kCheckScratchWords];

// In host code the symbol's name is only a host-side stand-in and must never
// be passed to a kernel; its device address is looked up on every call (the
// address belongs to the current context, which may change between calls;
// the lookup allocates nothing).

sqz_status fail(sqz_status st, const char* msg) {
    sqz_internal_set_last_error(msg);
    return st;
}

sqz_status cuda_fail(cudaError_t e, const char* what) {
    char buf[256];
    snprintf(buf, sizeof buf, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    (void)cudaGetLastError();
    return fail(SQZ_ERR_CUDA, buf);
}

// The scratch's device address in the current context, and the device.
sqz_status scratch_of_current_device(int** out, int* device) {
    cudaError_t e = cudaGetDevice(device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_check_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(check scratch)");
    *out = static_cast<int*>(p);
    return SQZ_OK;
}

}  // namespace

extern "C" SQZ_API sqz_status sqz_check_csr_static(const int32_t* rowptr, const int32_t* col, int32_t n_out,
                                                   int32_t k_in, int64_t nnz, void* stream, int32_t* flags) {
    if (!flags) return fail(SQZ_ERR_INVALID_ARG, "flags is NULL");
    *flags = 0;
    if (n_out < 0 || n_out == INT32_MAX || k_in < 0)
        return fail(SQZ_ERR_INVALID_ARG, "n_out must be in [0, 2^31-2] and k_in >= 0");
    if (nnz < 0 || nnz > INT32_MAX) return fail(SQZ_ERR_INVALID_ARG, "nnz must be in [0, 2^31-1] (int32 CSR indices)");
    if (nnz == 0) return SQZ_OK;  // like sqz_create_layer: nothing to check without outliers
    if (!rowptr || !col) return fail(SQZ_ERR_INVALID_ARG, "nnz > 0 but rowptr or col is NULL");

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The verdict is read back with a synchronisation, which a stream capture
    // cannot contain: refuse before touching the stream, so the caller's
    // capture stays intact.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone)
        return fail(SQZ_ERR_UNSUPPORTED, "the stream is being captured into a CUDA graph; the check reads its "
                                         "verdict back and synchronises, which a capture cannot contain");

    int* scratch = nullptr;
    int device = 0;
    sqz_status st = scratch_of_current_device(&scratch, &device);
    if (st != SQZ_OK) return st;
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) sms = 148;

    // The array keeps the previous call's flags: clear the word first.
    e = cudaMemsetAsync(scratch, 0, sizeof(int), s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the check scratch");
    const int64_t work = nnz > (int64_t)n_out + 1 ? nnz : (int64_t)n_out + 1;
    int64_t blocks = (work + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    sqz::validate_csr_kernel<<<(unsigned)blocks, 256, 0, s>>>(rowptr, col, n_out, k_in, nnz, scratch);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "CSR check launch");
    int h = 0;
    e = cudaMemcpyAsync(&h, scratch, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading the check result");
    *flags = h;
    return SQZ_OK;
}
