/*
 * sqz.h -- C ABI of the Dense-and-Sparse LUT-dequant GEMV library (libsqz.so)
 * for NVIDIA B200 (sm_100a).
 *
 * Operation ("SqueezeLLM: Dense-and-Sparse Quantization", summary page,
 * §3.4 "The Dense-and-Sparse Decomposition" and "Kernel Implementation"):
 *
 *     y = (Q + S) x
 *
 *   Q  dense part: every weight w(i,k) is a b-bit index (b = 3 or 4) into a
 *      lookup table of 2^b fp16 centroids owned by output row i
 *      (channel-wise LUTs, §3.2 "Sensitivity-Based K-Means Quantizer");
 *      w(i,k) = lut[i][code(i,k)].
 *   S  sparse outliers in CSR form: fp16 values, int32 column indices,
 *      int32 row pointer (§3.4 "The Sparse Matrix Storage Format").
 *   x  fp16 activations, batch 1..16; y fp16 outputs.
 *
 * Canonical storage (what sqz_create_layer reads):
 *   codes  uint32 [n_out][k_in*bits/32], one LSB-first bitstream per row:
 *          code(i,k) is the bits-wide field that starts at stream bit k*bits,
 *          stream bit p being bit (p mod 32) of word (p div 32) of row i.
 *          Exactly `bits` bits per index, no padding (§3.4 "The 3/4-bit
 *          storage format": eight 3-bit indices in 3 bytes).  For 3-bit codes
 *          this is the same as groups of 32 codes in 3 words; codes 10 and
 *          21 of every group straddle two words.
 *   lut    uint16 (fp16 bit patterns) [n_out][2^bits]
 *   rowptr int32 [n_out+1], col int32 [nnz], val uint16 (fp16 bits) [nnz].
 *          Columns within a row may be unsorted; duplicates are summed;
 *          empty rows are allowed.  Q and S are added: a position present
 *          in S still has a code in Q.
 *
 * Arithmetic: products of fp16 operands are exact in fp32; accumulation is
 * in fp32; y(i,b) is rounded once to fp16 (round to nearest even).  The
 * result agrees with the exact value within
 * 1e-3 * (sum_k |w(i,k) x(b,k)| + sum_j |val(j) x(b,col(j))|) + 1e-6 (j over
 * row i's outliers) and is bitwise reproducible from run to run (no
 * floating-point atomics).
 *
 * Layouts: x is [batch][ldx] and y is [batch][ldy], row-major (the
 * torch `x @ W.T` convention).  y is overwritten, never accumulated into.
 *
 * Errors: every entry point returns an sqz_status; nothing throws, aborts or
 * traps.  sqz_last_error() gives a message for the last non-OK status of the
 * calling thread.
 */
#ifndef SQZ_H_
#define SQZ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points keep default visibility even when the library is
 * built with -fvisibility=hidden. */
#if defined(__GNUC__)
#define SQZ_API __attribute__((visibility("default")))
#else
#define SQZ_API
#endif

typedef struct sqz_layer* sqz_layer_t;

typedef enum {
    SQZ_OK = 0,
    SQZ_ERR_INVALID_ARG = 1, /* null pointer, bad size, malformed CSR          */
    SQZ_ERR_UNSUPPORTED = 2, /* valid request this build does not implement    */
    SQZ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed    */
    SQZ_ERR_OOM = 4,         /* device allocation failed                       */
    SQZ_ERR_TIMEOUT = 5      /* a bounded device wait gave up                  */
} sqz_status;

/* Largest batch (columns of x) one call accepts. */
#define SQZ_MAX_BATCH 16

/* Description of one layer in canonical storage.  All pointers are DEVICE
 * pointers on the current CUDA device, owned by the caller. */
typedef struct {
    int32_t n_out;          /* N: output rows, >= 0                                   */
    int32_t k_in;           /* K: input columns, >= 0; K % 32 == 0 for 3-bit,
                               K % 8 == 0 for 4-bit (whole 32-bit words per row)      */
    int32_t bits;           /* 3 or 4                                                 */
    const uint32_t* codes;  /* [n_out][k_in*bits/32]; may be NULL when N*K == 0        */
    const uint16_t* lut;    /* [n_out][1<<bits] fp16 bits; may be NULL when N == 0     */
    int64_t nnz;            /* outliers, 0 <= nnz <= INT32_MAX - 64                   */
    const int32_t* rowptr;  /* [n_out+1]; may be NULL when nnz == 0                   */
    const int32_t* col;     /* [nnz];     may be NULL when nnz == 0                   */
    const uint16_t* val;    /* [nnz] fp16 bits; may be NULL when nnz == 0             */
} sqz_layer_desc;

/*
 * Build a layer handle from canonical storage: the per-layer output of the
 * offline compression pipeline (codes, LUTs and outlier matrix; §3.2
 * "Big-Picture Architecture"), which the inference kernels consume.
 *
 * Copies every array into device memory the handle owns, rearranged into
 * the kernels' layout; the caller may free its arrays once this returns.
 * Work is ordered on `stream` (a cudaStream_t; NULL = legacy default
 * stream) and the call synchronises that stream once to read the CSR
 * validation result.
 *
 * Errors: SQZ_ERR_INVALID_ARG for a NULL desc/out, bits not in {3,4}, K not
 * a whole number of words per row, negative sizes, a required NULL array,
 * or a CSR that fails the device-side check (rowptr[0] != 0, rowptr
 * decreasing, rowptr[N] != nnz, a column outside [0, K)); SQZ_ERR_OOM;
 * SQZ_ERR_CUDA.  On error *out is set to NULL and nothing is leaked.
 */
SQZ_API sqz_status sqz_create_layer(const sqz_layer_desc* desc, void* stream, sqz_layer_t* out);

/*
 * y = (Q + S) x for `batch` columns, asynchronously on `stream`.
 *
 * x: device, fp16 bits, [batch][ldx] (ldx >= K); y: device, fp16 bits,
 * [batch][ldy] (ldy >= N).  x and y are borrowed until the stream reaches
 * the end of this call; they must not overlap.  One fused kernel launch:
 * the dense LUT part and the CSR part of a row are summed on chip and y is
 * written once (§3.4 "Kernel fusion").
 *
 * Errors: SQZ_ERR_INVALID_ARG (NULL layer/x/y with non-empty sizes, batch
 * outside [1, SQZ_MAX_BATCH], ldx < K, ldy < N); SQZ_ERR_CUDA if the launch
 * fails.  No synchronisation.
 */
SQZ_API sqz_status sqz_gemv(sqz_layer_t layer, const uint16_t* x, int32_t batch, int64_t ldx, uint16_t* y,
                    int64_t ldy, void* stream);

/*
 * The same product for callers whose activations live in HOST memory:
 * x (host, [batch][ldx]) in, y (host, [batch][ldy]) out; synchronises
 * `stream` before returning.  x is copied to the handle's device staging
 * buffer with cudaMemcpyAsync (asynchronous when x is page-locked).  A
 * page-locked y (cudaHostAlloc / cudaMallocHost / cudaHostRegister,
 * including torch's pin_memory) is written by the product kernel's own
 * stores through the buffer's device mapping, without a copy back; a
 * pageable y is written to a staging buffer and copied back.  With both
 * buffers page-locked on a created (non-default) stream, the copy and the
 * product are captured as a CUDA graph on first use and replayed by later
 * calls with the same buffers, shape and stream (up to 64 per handle, least
 * recently used dropped; released by sqz_destroy and by a change of the
 * handle's MAC unit, CSR mode or decode-ahead setting).  Elements of y
 * beyond column N of each row are not written.  Not thread-safe against
 * other calls on the same handle.  Errors as sqz_gemv.
 */
SQZ_API sqz_status sqz_gemv_host(sqz_layer_t layer, const uint16_t* x_host, int32_t batch, int64_t ldx,
                         uint16_t* y_host, int64_t ldy, void* stream);

/*
 * Write the dequantized dense weights w(i,k) = lut[i][code(i,k)] as fp16 bit
 * patterns to w_out (device, [n_out][k_in]), decoded from the handle's
 * internal layout with the same decoder the GEMV kernel uses.  For
 * checking only (the GEMV never materialises these weights).  Async on
 * `stream`.  Errors: SQZ_ERR_INVALID_ARG, SQZ_ERR_CUDA.
 */
SQZ_API sqz_status sqz_debug_dequant(sqz_layer_t layer, uint16_t* w_out, void* stream);

/* Multiply-accumulate unit of the fused kernel (sqz_layer_set_mac). */
#define SQZ_MAC_TENSOR_CORES 0 /* mma.sync m16n8k16, fp32 accumulate (default)        */
#define SQZ_MAC_CUDA_CORES 1   /* fma.rn.f32.f16 on the CUDA cores, batch 1 only     */
#define SQZ_MAC_MIXED 2        /* even k16-steps on the tensor cores, odd steps on   */
                               /* the CUDA cores, batch 1 only                       */

/*
 * Choose the unit that performs the multiply-accumulates of the dense part.
 * All give results within the same bound (fp16 products are exact in fp32,
 * accumulation is fp32; only the order of the additions differs); the
 * choice applies to batch-1 calls, larger batches always use the tensor
 * cores.  Not thread-safe against concurrent sqz_gemv calls on the same
 * handle.
 * Errors: SQZ_ERR_INVALID_ARG.
 */
SQZ_API sqz_status sqz_layer_set_mac(sqz_layer_t layer, int32_t mac);

/* How the fused kernel sums the outliers (sqz_layer_set_csr_mode). */
#define SQZ_CSR_BALANCED 0 /* equal nonzero shares per thread, pieces combined per row (default) */
#define SQZ_CSR_ROWWISE 1  /* each row's nonzeros summed by one thread: the plain CSR SpMV     */

/*
 * Choose the sparse scheme ("SqueezeLLM: Dense-and-Sparse Quantization",
 * summary page, §3.4 "Balanced Sparse Kernel": the balanced split against
 * the plain row-per-thread CSR kernel it replaces).  Both give results
 * within the same bound (only the order of the additions differs); the
 * row-wise scheme exists to compare the two on skewed outlier
 * distributions, where its cost follows the longest row of a tile.  In
 * row-wise mode the dense part always uses the tensor cores (the
 * sqz_layer_set_mac choice applies to the balanced mode).  Not
 * thread-safe against concurrent sqz_gemv calls on the same handle.
 * Errors: SQZ_ERR_INVALID_ARG.
 */
SQZ_API sqz_status sqz_layer_set_csr_mode(sqz_layer_t layer, int32_t mode);

/*
 * The decode-ahead kernel (batches of 1..8 columns; off by default): every
 * warp decodes its first code units into tensor memory while the call waits
 * for the previous kernel of the stream and for x, and multiplies them once x
 * has arrived.  enable = 1 takes it (two CTAs of 8 dense warps per SM when
 * they fit half an SM, else one CTA of 16); 8 or 16 ask for one of the two
 * CTA shapes; 0 (the default) takes the 12-warp kernel.  All choices give
 * results within the same bound, and the two decode-ahead shapes give the
 * same bits.  In a chain of dependent calls the next call's decoding ahead
 * runs while the current call computes, so on B200 it has not been faster
 * than the default; it applies with the default MAC unit and CSR mode.  Not
 * thread-safe against concurrent sqz_gemv calls on the same handle.
 * Errors: SQZ_ERR_INVALID_ARG (enable not in {0, 1, 8, 16}).
 */
SQZ_API sqz_status sqz_layer_set_predecode(sqz_layer_t layer, int32_t enable);

/*
 * Read and clear the handle's device status word, ordered on `stream`
 * (synchronises it).  *status receives the word: 0 means every call so far
 * completed normally; bit 0 (1) means a bounded wait for a copy into shared
 * memory gave up, and then y of the affected call is undefined.  Returns
 * SQZ_ERR_TIMEOUT (with *status set) when bit 0 was set, so that a caller
 * checking only return codes sees it; SQZ_OK otherwise.
 * Errors: SQZ_ERR_INVALID_ARG, SQZ_ERR_CUDA, SQZ_ERR_TIMEOUT.
 */
SQZ_API sqz_status sqz_layer_status(sqz_layer_t layer, void* stream, int32_t* status);

/* Sizes of a handle (any output pointer may be NULL). */
SQZ_API sqz_status sqz_layer_info(sqz_layer_t layer, int32_t* n_out, int32_t* k_in, int32_t* bits, int64_t* nnz,
                          int64_t* device_bytes);

/*
 * The launch plan sqz_gemv would use for a layer shape and batch on a device
 * with the given SM count and shared memory (per SM, and the opt-in maximum
 * of one CTA) -- computed on the host, no device needed -- for the even split
 * of row tiles over the CTAs (a layer whose outliers are skewed enough to be
 * split by weight, see sqz_tile_split_query, gives some CTAs up to twice the
 * tiles, and its plan sizes their shared memory for that).  fused = 0 means the
 * row-per-warp kernel serves the call (all other fields 0).  Otherwise the
 * batch runs as `launches` launches of up to columns_per_launch columns,
 * each a grid of `grid` CTAs of `threads` threads with smem_bytes of dynamic
 * shared memory (ctas_per_sm = 2 when two CTAs share an SM), x staged in
 * `passes` chunks of K, a code ring of ring_stages stages per warp and up to
 * csr_stage_entries outliers per CTA staged in shared memory (the first
 * launch's plan; a shorter last launch may differ).  `predecode` is the
 * handle's sqz_layer_set_predecode choice (0, 1, 8 or 16); out->predecode = 1 when
 * the call takes the decode-ahead kernel (the query assumes the default MAC
 * unit and CSR mode).  No counterpart in the paper: it exposes this
 * library's own scheduling.
 * Errors: SQZ_ERR_INVALID_ARG for a NULL out, bits not in {3,4}, n_out or k_in
 * < 1, batch outside [1,16], or a non-positive device figure.
 */
typedef struct {
    int32_t fused, columns_per_launch, launches, grid, threads, ctas_per_sm, smem_bytes, passes, ring_stages,
        csr_stage_entries, predecode;
} sqz_plan_info;
SQZ_API sqz_status sqz_plan_query(int32_t n_out, int32_t k_in, int32_t bits, int32_t batch, int32_t sm_count,
                                  int32_t smem_per_sm, int32_t smem_optin, int32_t predecode, sqz_plan_info* out);

/*
 * The split of a layer's row tiles (16 rows each) over the fused kernel's
 * CTAs that sqz_create_layer computes from the outlier matrix, computed on
 * the host from a HOST copy of rowptr ([n_out + 1] int32, rowptr[0] = 0,
 * non-decreasing) -- no device needed.  The balanced sparse kernel of the
 * summary page (§3.4 "Kernel Implementation", "Balanced sparse kernel")
 * gives each thread an equal share of nonzeros; when the outliers are skewed
 * over the rows, this library also balances across CTAs: each tile weighs
 * w x its 256-column units + its nonzeros (w = 100 at 3 bits, 150 at 4),
 * and the CTAs take consecutive runs of 1 to twice the even count of tiles,
 * cut so that the heaviest run is as light as possible.  That split is
 * used only when it lowers the heaviest CTA's weight by more than 5 %.
 * On return first[c] (c = 0..grid, grid = min(sm_count, tiles)) is the first
 * tile of CTA c and first[grid] the tile count; *weighted = 1 when the split
 * by weight is used, 0 for the even split (runs differing by at most one
 * tile).  `first` is caller-owned host memory of at least grid + 1 entries.
 * Errors: SQZ_ERR_INVALID_ARG for NULL pointers, bits not in {3,4}, n_out,
 * k_in or sm_count < 1, or a rowptr that does not start at 0 or decreases.
 */
SQZ_API sqz_status sqz_tile_split_query(const int32_t* rowptr, int32_t n_out, int32_t k_in, int32_t bits,
                                        int32_t sm_count, int32_t* first, int32_t* weighted);

/* Release a handle and its device memory.  NULL is accepted.  The caller
 * must make sure no work that uses the handle is still in flight. */
SQZ_API sqz_status sqz_destroy(sqz_layer_t layer);

/*
 * fp16 dense matrix-vector product y = W x with W fp16 [n_out][ldw] (ldw >=
 * k_in), x [batch][ldx], y [batch][ldy]: the uncompressed fp16 baseline that
 * the quantized kernels' speedups are reported against (§5 "Inference
 * Latency and Memory Benchmarking", Table G.12), used here as a bandwidth
 * yardstick.  Same arithmetic contract and errors as sqz_gemv.
 */
SQZ_API sqz_status sqz_fp16_gemv(const uint16_t* w, int32_t n_out, int32_t k_in, int64_t ldw, const uint16_t* x,
                         int32_t batch, int64_t ldx, uint16_t* y, int64_t ldy, void* stream);

/*
 * Check an outlier matrix in CSR form exactly as sqz_create_layer does,
 * without allocating any device memory.  (This entry point has no
 * counterpart in the paper; it exists for callers that cannot allocate.)
 *
 * Who needs it: code that cannot call cudaMalloc where it wants the check --
 * serving loops that must not take the implicit device synchronisation of
 * cudaMalloc/cudaFree, and runtimes that reserve all device memory up front
 * and forbid later allocations.  sqz_create_layer allocates a flag word for
 * its check; this call uses a fixed 256-byte device array inside the library
 * instead (held on every GPU that loads the library until the process exits;
 * the check uses one 4-byte word of it whatever the matrix size).
 *
 * rowptr: device [n_out+1]; col: device [nnz] (both caller-owned, read
 * only).  *flags (host) receives 0 for a well-formed matrix, else the OR of
 * 1 rowptr[0] != 0, 2 rowptr[n_out] != nnz, 4 rowptr decreasing, 8 a column
 * outside [0, k_in).  nnz == 0 writes 0 without touching the device (as
 * sqz_create_layer ignores the CSR arrays then).  The call is ordered on
 * `stream` and synchronises it before returning, so it cannot be recorded
 * into a CUDA graph: on a stream that is being captured it returns
 * SQZ_ERR_UNSUPPORTED before enqueuing anything (the capture stays valid).
 *
 * Every call looks up the array's device address in the current context
 * (no allocation) and clears the flag word first.  Every call shares the one
 * array: calls whose work overlaps on the GPU (different streams, or host
 * threads) race and may report each other's flags -- serialise them.
 *
 * Errors: SQZ_ERR_INVALID_ARG for a NULL flags pointer, n_out outside
 * [0, 2^31-2], k_in < 0, nnz outside [0, 2^31-1] (the int32 limits of the
 * CSR format), or NULL rowptr/col with nnz > 0; SQZ_ERR_UNSUPPORTED on a
 * stream under capture; SQZ_ERR_CUDA.  Never calls cudaMalloc or cudaFree.
 */
SQZ_API sqz_status sqz_check_csr_static(const int32_t* rowptr, const int32_t* col, int32_t n_out, int32_t k_in,
                                        int64_t nnz, void* stream, int32_t* flags);

/* ------------------------------------------------------------ encoder ---
 * Quantize an fp16 weight matrix into the layer format sqz_create_layer
 * takes ("SqueezeLLM: Dense-and-Sparse Quantization", summary page:
 * "The Dense-and-Sparse Decomposition", W = D + S with S the weights beyond
 * two percentile thresholds, kept exactly in CSR; "Sensitivity-Based
 * Non-Uniform Quantization", Eq. 1: per output row a 1-D k-means over the
 * row's values gives the 2^bits centroids of the row's LUT, each weight is
 * stored as the index of its centroid; the sensitivity weighting, which
 * needs gradients of a real model, is not part of it).
 *
 * Definition (every step exact, so the result is unique):
 *   - m = floor(outlier_fraction * n_out * k_in / 2 + 1/2), at most half
 *     the weights; the outliers are the first m and the last m weights in
 *     ascending order of (value, row-major position), -0 and +0 being one
 *     value (the 0.2th/99.8th percentiles of the page are fraction 0.004);
 *   - D = W with the outliers set to +0; per row of D, k-means with
 *     2^bits centroids starting from the uniform grid over [min, max] of the
 *     row; each Lloyd iteration assigns every value to its nearest centroid
 *     (|d - c_j| in fp64, the lowest j on a tie) and moves each centroid to
 *     the mean of its values (an empty centroid stays); it stops when no
 *     centroid moves or after max_iters iterations;
 *   - lut = the centroids rounded to fp16 (nearest, ties to even); each
 *     weight's code = its nearest lut entry (lowest index on a tie), packed
 *     as sqz_layer_desc.codes (canonical LSB-first bitstream).
 *
 * w: device fp16 bits [n_out][k_in], row-major, read only.  Outputs
 * (device, caller-owned): codes [n_out][k_in*bits/32], lut [n_out][2^bits],
 * rowptr [n_out+1], col and val [nnz_capacity] (NULL allowed when no
 * outliers are asked for), iters_out [n_out] (may be NULL: the iterations
 * each row ran).  *nnz_out (host) receives the number of outliers, which is
 * sqz_encode_outliers(n_out * k_in, outlier_fraction) -- size col/val with it.
 * The call is ordered on `stream`, allocates a device workspace of about
 * n_out*k_in bytes, and synchronises the stream before returning.
 *
 * Errors: SQZ_ERR_INVALID_ARG for NULL w/codes/lut/rowptr/nnz_out, bits not
 * in {3,4}, n_out or k_in < 1, k_in not a multiple of 32 (3-bit) or 8 (4-bit),
 * outlier_fraction outside [0,1], max_iters outside [0,100000], nnz_capacity
 * below the outlier count, NULL col/val with outliers, or weights that are
 * inf or NaN; SQZ_ERR_UNSUPPORTED when k_in * max|w| reaches 2^29 (row sums of
 * fp16 values are then no longer exact in fp64), k_in exceeds 102400 (a row
 * is staged in 200 KB of shared memory) or the outliers exceed the int32
 * range; SQZ_ERR_OOM; SQZ_ERR_CUDA.
 */
SQZ_API sqz_status sqz_encode(const uint16_t* w, int32_t n_out, int32_t k_in, int32_t bits, double outlier_fraction,
                              int32_t max_iters, uint32_t* codes, uint16_t* lut, int32_t* rowptr, int32_t* col,
                              uint16_t* val, int64_t nnz_capacity, int64_t* nnz_out, int32_t* iters_out,
                              void* stream);

/* Outliers sqz_encode selects for n_weights weights at outlier_fraction
 * (2*m above; 0 for n_weights <= 0 or a negative or NaN fraction). */
SQZ_API int64_t sqz_encode_outliers(int64_t n_weights, double outlier_fraction);

/* Message for the calling thread's last non-OK status ("" if none). */
SQZ_API const char* sqz_last_error(void);

/* Library version: major*10000 + minor*100 + patch. */
SQZ_API int32_t sqz_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQZ_H_ */
