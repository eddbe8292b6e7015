/*
 * ss1.h -- C ABI of the SS1 (Sketch Structured Transform) linear-layer forward on B200.
 *
 * The operation. "SS1: Accelerating Inference with Fast and Expressive Sketch Structured
 * Transform" (atlas.scime.ai paper summary), section "Approach": random parameter sharing is
 * confined to one neuron's weight vector through K- and N-coalescing hash functions; the
 * input is first sketched (reduced by the compression factor c through signed additions)
 * and then multiplied with the compressed weights. With N-blocks of BN neurons
 * (nb = n / BN) and K-chunks of BK inputs (kc = k / BK), every (nb, kc) has its own hash
 * h_nb mapping the chunk onto S = BK / c slots, exactly c inputs per slot, and signs
 * g_nb = +-1. Compressed column j = kc * S + slot. The layer computes
 *
 *     Y[m, n] = sum_k X[m, k] * g_nb(k) * Wc[n, h_nb(k)],    nb = n / BN,
 *
 * by sketching Xs_nb[m, j] = sum_{k : h_nb(k) = j} g_nb(k) X[m, k] on chip and
 * multiplying Y[:, block nb] = Xs_nb Wc[block nb, :]^T. No bias, no activation.
 *
 * The hash (the pages leave its family open; this library fixes it). For block id
 * b = nb * KC + kc (KC = K / BK): key = seed XOR mix64(b + 1), where mix64 is the SplitMix64
 * finaliser (Steele, Lea & Flood, OOPSLA 2014); draw t = mix64(key + (t+1) * 0x9E3779B97F4A7C15).
 * A Fisher-Yates (Durstenfeld) shuffle of [0, BK) takes draws t = 0 .. BK-2 for positions
 * i = BK-1 .. 1 with j = ((draw >> 32) * (i + 1)) >> 32; signs g(k) = -1 if bit 63 of draw
 * BK-1+k is set; slot(k) = perm[k] mod S. c = 1 is the identity hash with all signs +1.
 *
 * Conventions for every entry point:
 *  - Returns an int status (SS1_OK or a negative SS1_ERR_*). Never aborts, exits or prints.
 *  - Device pointers are plain CUDA device addresses on the handle's device; host pointers
 *    are plain host memory. All matrices are dense row-major with no padding.
 *  - Nothing here synchronises the device unless stated.
 */
#ifndef SS1_H
#define SS1_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SS1_API __attribute__((visibility("default")))
#else
#define SS1_API
#endif

/* Opaque layer handle: owns the device hash tables of one (K, N, c, BK, BN, seed). */
typedef struct ss1_layer* ss1_handle;

/* Element type of X, Wc and Y. Accumulation is fp32 in both cases. */
enum ss1_dtype { SS1_DTYPE_BF16 = 0, SS1_DTYPE_FP32 = 1 };

/* Kernel choice for ss1_forward_with. AUTO is what ss1_forward uses. */
enum ss1_kernel {
    SS1_KERNEL_AUTO = 0,
    SS1_KERNEL_TC = 1,      /* bf16: TMA + on-chip sketch + tcgen05/TMEM tensor-core GEMM */
    SS1_KERNEL_SIMT = 2,    /* bf16 or fp32: CUDA-core sketch + FMA GEMM, any valid shape */
    SS1_KERNEL_SMALLM = 3   /* bf16, decode-sized M: streams Wc once (tensor cores for BN = 128) */
};

enum ss1_status {
    SS1_OK = 0,
    SS1_ERR_INVALID_ARG = -1,        /* a size, dtype, kernel or shape precondition failed   */
    SS1_ERR_UNSUPPORTED_DEVICE = -2, /* current device is not sm_100 (B200 class)             */
    SS1_ERR_CUDA = -3,               /* a CUDA runtime call or kernel launch failed           */
    SS1_ERR_OUT_OF_MEMORY = -4,      /* device or pinned allocation failed in ss1_create      */
    SS1_ERR_MISALIGNED = -5,         /* a pointer is not 16-byte aligned                      */
    SS1_ERR_DEVICE_TIMEOUT = -6,     /* a kernel gave up a bounded wait (see ss1_device_status)*/
    SS1_ERR_BAD_HANDLE = -7,         /* null or destroyed handle                              */
    SS1_ERR_UNSUPPORTED_SHAPE = -8   /* this kernel cannot run this shape (choose another)    */
};

/*
 * ss1_create -- build the hash and sign tables of one SS1 layer on the current device.
 *   K, N   : input and output features, K >= 1, N >= 1.
 *   c      : compression factor, one of 1, 2, 4, 8. Wc has K / c columns.
 *   BK, BN : K-chunk and N-block sizes; K % BK == 0, N % BN == 0, BK % c == 0, BK <= 256,
 *            BN % 16 == 0, and (N / BN) * K < 2^31 table entries.
 *   seed   : table seed (any 64-bit value).
 *   out    : receives the handle (host pointer to a handle variable).
 * Allocates device memory and one pinned host word (device status), launches the table
 * generator and synchronises. The device memory is the tables (17 bytes per (N / BN) * K
 * entry). Where BN == 128 and N / BN is at most the SM count, it is also the decode kernel's
 * K-split scratch: 2 x SMs x 32 KiB of fp32 partials plus 16 bytes per N-block of counters.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, OUT_OF_MEMORY, CUDA. On error *out is set to NULL
 * and nothing is leaked.
 */
SS1_API int ss1_create(int64_t K, int64_t N, int c, int BK, int BN, uint64_t seed, ss1_handle* out);

/*
 * ss1_forward -- Y = SS1(X) with compressed weights Wc, enqueued on `stream`.
 *   X  : device, [M, K] of `dtype`.       Wc : device, [N, K / c] of `dtype`.
 *   Y  : device, [M, N] of `dtype`, written in full; must not overlap X or Wc.
 *   M  : rows, M >= 0 (M == 0 is a no-op).
 *   dtype  : SS1_DTYPE_BF16 or SS1_DTYPE_FP32.
 *   stream : a cudaStream_t passed as void* (NULL = legacy default stream).
 * The caller owns X, Wc and Y and keeps them alive until the stream work completes.
 * Asynchronous: returns after the launch. Errors: BAD_HANDLE, INVALID_ARG, MISALIGNED
 * (X, Wc, Y must be 16-byte aligned), CUDA (launch failure), DEVICE_TIMEOUT (an earlier
 * launch on this handle reported a bounded-wait time-out; see ss1_device_status).
 * Decode calls (the SMALLM kernel, which AUTO picks for M <= 16) on a handle with N-blocks of
 * 128 pass partial sums through the handle's K-split scratch: such calls on one handle must not
 * overlap on the device (order them on one stream or with events). Every other call only reads
 * the handle, so those may run concurrently on any streams.
 * The tensor-core decode kernel is launched with programmatic dependent launch: it may start
 * while the previous kernel on the stream is still running, but before that kernel completes it
 * only prefetches Wc into L2. It reads X and the tables and writes Y only afterwards, so stream
 * order holds as for any launch.
 */
SS1_API int ss1_forward(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M, int dtype,
                        void* stream);

/*
 * ss1_forward_with -- ss1_forward with an explicit kernel (enum ss1_kernel). Same arguments,
 * ownership and errors; additionally UNSUPPORTED_SHAPE when the chosen kernel cannot run this
 * (dtype, M, shape): TC needs bf16, BK one of 64, 128, 256, S = BK / c a multiple of 16,
 * BN == 128, and K, K / c multiples of 8;
 * SMALLM needs bf16, M <= 64 and K, K / c multiples of 8, and either BN == 128 (the
 * tensor-core decode kernel) or S = BK / c a power of two >= 8 with BN a multiple of 8 (the
 * CUDA-core one); SIMT runs every valid shape.
 */
SS1_API int ss1_forward_with(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M, int dtype,
                             int kernel, void* stream);

/*
 * ss1_select_kernel -- the kernel ss1_forward would use for (M, dtype); writes it to *kernel.
 */
SS1_API int ss1_select_kernel(ss1_handle h, int64_t M, int dtype, int* kernel);

/*
 * ss1_destroy -- free the handle's tables. Synchronises the device first, so work already
 * enqueued with this handle finishes. NULL is accepted (returns OK).
 */
SS1_API int ss1_destroy(ss1_handle h);

/*
 * ss1_get_tables -- copy the canonical tables to host memory (synchronous; for checking).
 *   h_host : host int32 [N / BN, K]: compressed column kc * S + slot of input k in block nb.
 *   g_host : host int8  [N / BN, K]: sign (+1 / -1) of input k in block nb.
 * Either pointer may be NULL to skip it. Errors: BAD_HANDLE, CUDA.
 */
SS1_API int ss1_get_tables(ss1_handle h, int32_t* h_host, int8_t* g_host);

/* ss1_get_info -- the layer's parameters (any output pointer may be NULL). */
SS1_API int ss1_get_info(ss1_handle h, int64_t* K, int64_t* N, int* c, int* BK, int* BN);

/*
 * ss1_device_status -- read (and clear) the handle's device status word without
 * synchronising. Kernels with bounded waits write a non-zero code there instead of
 * trapping when a wait runs out; the word lives in pinned host memory. Returns SS1_OK or
 * SS1_ERR_DEVICE_TIMEOUT; *detail (may be NULL) receives the raw code (kernel id and wait site).
 * Call after synchronising the stream to see the result of the work enqueued so far. When it
 * reports a time-out it also synchronises the device and resets the decode kernel's K-split
 * counters, which a launch that gave up may have left non-zero.
 */
SS1_API int ss1_device_status(ss1_handle h, int32_t* detail);

/* ss1_strerror -- static, NUL-terminated text for a status code. */
SS1_API const char* ss1_strerror(int status);

/* Table entries ((N / BN) * K) that ss1_forward_noalloc accepts at most. */
#define SS1_NOALLOC_MAX_ENTRIES 983040

/*
 * ss1_forward_noalloc -- ss1_create + ss1_forward in one call that allocates nothing.
 * This entry point has no counterpart in the SS1 paper; it only changes where the layer's
 * hash tables live. It is for callers that must not let a library allocate device memory:
 * a serving process that reserves all device memory for its own pool up front (an
 * allocation could fail or fragment that pool mid-run), or code that needs one layer once
 * and cannot afford ss1_create's allocations and device synchronisation.
 *
 *   K, N, c, BK, BN, seed : as for ss1_create (same checks, same tables, same Y).
 *   X, Wc, Y, M, dtype    : as for ss1_forward.
 *   device_status : device int32 word owned by the caller, or NULL. The call clears it on
 *                   `stream` before the launches; a kernel that gives up a bounded wait
 *                   writes its non-zero code there (read it after synchronising). With
 *                   NULL the library's own word is used and a time-out is not reported.
 *   stream        : a cudaStream_t passed as void* (NULL = legacy default stream).
 *
 * Every call regenerates the tables on `stream` into one fixed region of device memory
 * that the library reserves statically (16 MiB per device: 17 bytes per table entry plus
 * padding), then runs the kernel ss1_forward would choose. The decode-sized path (M <= 64)
 * splits K across CTAs as it does for a handle, with a second static region of 12 MiB for the
 * fp32 partials and 3 KiB of arrival counters; the call clears those counters on `stream`.
 * Shapes with (N / BN) * K > SS1_NOALLOC_MAX_ENTRIES are rejected with UNSUPPORTED_SHAPE. No
 * cudaMalloc, cudaFree, pinned allocation or allocating library routine is called, and
 * nothing synchronises the device; the tables need no zeroing because the table kernels
 * write all of them that the forward reads.
 *
 * The first call on a device does one-time set-up (it looks up the region's address and
 * sets kernel attributes); make that first call outside any stream capture.
 * Calls share the one region: two calls whose work can overlap on the device (different
 * streams without ordering, or different host threads) race on the tables and give wrong
 * results. Order them on one stream or with events. Asynchronous: returns after the
 * launches. Errors: INVALID_ARG, UNSUPPORTED_DEVICE, UNSUPPORTED_SHAPE, MISALIGNED (X, Wc,
 * Y and device_status must be 16- resp. 4-byte aligned), CUDA.
 */
SS1_API int ss1_forward_noalloc(int64_t K, int64_t N, int c, int BK, int BN, uint64_t seed, const void* X,
                                const void* Wc, void* Y, int64_t M, int dtype, int32_t* device_status,
                                void* stream);

/*
 * ss1_test_device_timeout -- exercises the bounded-wait error path without a fault, for tests of
 * failure handling (the SS1 pages have no counterpart). Launches one thread on `stream` that
 * waits on a barrier nothing completes, with the forward kernels' bounded wait cut to
 * limit_ns nanoseconds (1 .. 2e9). When the limit passes, the thread writes the handle's status
 * word as a stalled forward kernel would: kernel id 3, site 1, that is (3 << 8) | 0x81. Then it
 * returns, and the context stays usable. Afterwards ss1_forward on this handle returns
 * SS1_ERR_DEVICE_TIMEOUT until ss1_device_status has read and cleared the word.
 * Asynchronous. Errors: BAD_HANDLE, INVALID_ARG (limit_ns out of range), CUDA (launch failure).
 */
SS1_API int ss1_test_device_timeout(ss1_handle h, int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SS1_H */
