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

#include <stddef.h>
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

/* Activation of the fused epilogue (ss1_forward_ex, ss1_chain_forward). */
enum ss1_activation {
    SS1_ACT_NONE = 0,
    SS1_ACT_RELU = 1,   /* max(v, 0)                                       */
    SS1_ACT_GELU = 2    /* v * Phi(v) = 0.5 v (1 + erf(v / sqrt(2))), exact */
};

/* Layers that one ss1_chain_forward call takes at most. */
#define SS1_CHAIN_MAX_LAYERS 4

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
 * entry); after this call the handle is only read.
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
 * Re-entrant: every kernel only reads the handle and writes nothing but Y (the decode kernel's
 * K-split partial sums stay in the shared memory of one thread-block cluster), so calls on one
 * handle may run concurrently on any streams and threads.
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
 * Call after synchronising the stream to see the result of the work enqueued so far.
 */
SS1_API int ss1_device_status(ss1_handle h, int32_t* detail);

/* ss1_strerror -- static, NUL-terminated text for a status code. */
SS1_API const char* ss1_strerror(int status);

/*
 * ss1_forward_ex -- Y = act(SS1(X) + bias): the layer with a per-neuron bias and an activation.
 * "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
 * "Measured effects": SS1 layers replace the layers of the DLRM MLPerf top MLP; an MLP adds a
 * bias and an activation to each layer, which the pages leave to the model.
 *   bias : device, [N] of `dtype`, or NULL (no bias).   act : enum ss1_activation.
 *   kernel : enum ss1_kernel (AUTO picks as ss1_forward does). Other arguments as ss1_forward.
 * The tensor-core kernel for c >= 2 (every large-M bf16 layer of the workloads) adds the bias
 * and applies the activation to the fp32 sum in its epilogue, then rounds once; the other
 * kernels write Y and one elementwise pass follows (a second rounding for bf16).
 * Errors: as ss1_forward_with; INVALID_ARG for an unknown act; MISALIGNED for a bias not
 * aligned to its element.
 */
SS1_API int ss1_forward_ex(ss1_handle h, const void* X, const void* Wc, const void* bias, int act, void* Y, int64_t M,
                           int dtype, int kernel, void* stream);

/*
 * ss1_chain_forward -- a chain of bf16 SS1 layers, each the input of the next (an MLP):
 *   Y[0] = act[0](SS1_0(X) + bias[0]),  Y[l] = act[l](SS1_l(Y[l - 1]) + bias[l]).
 * Same source as ss1_forward_ex (the DLRM top MLP of "Measured effects").
 *   layers : n_layers (1 .. SS1_CHAIN_MAX_LAYERS) handles; K of layer l + 1 == N of layer l.
 *   X : device bf16 [M, K of layer 0].   Wc[l] : device bf16 [N_l, K_l / c_l].
 *   bias : NULL, or an array of n_layers device pointers (bf16 [N_l], each may be NULL).
 *   act : NULL (no activation), or n_layers enum ss1_activation values.
 *   Y : n_layers device pointers, Y[l] bf16 [M, N_l], all written (the caller owns them; the
 *       intermediate outputs are kept, as an MLP's backward pass needs them).
 * When every layer runs on the tensor-core kernel for c >= 2 with one (BK, c) and the same
 * N-block grouping (ss1_chain_fused says whether), the whole chain is one persistent launch:
 * each CTA carries whole 128-row tiles through every layer in order, so no layer waits for
 * another CTA. Otherwise the layers run one ss1_forward_ex after another. Asynchronous.
 * Errors: BAD_HANDLE, INVALID_ARG (sizes, NULL, act), MISALIGNED (X, Wc, Y 16-byte, bias 2-byte),
 * CUDA, DEVICE_TIMEOUT.
 */
SS1_API int ss1_chain_forward(const ss1_handle* layers, int n_layers, const void* X, const void* const* Wc,
                              const void* const* bias, const int* act, void* const* Y, int64_t M, void* stream);

/* ss1_chain_fused -- *fused = 1 if ss1_chain_forward runs these layers as one launch, else 0. */
SS1_API int ss1_chain_fused(const ss1_handle* layers, int n_layers, int* fused);

/*
 * ss1_project -- the SS1 weights closest to a dense weight: Wc = argmin || W_full(Wc) - W ||_F.
 * "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
 * "Key results": pre-trained dense layers (BERT-Base, Llama-3-8B) are projected onto SS1. The
 * pages give no formula; this is the orthogonal projection onto the tied weights of this
 * handle's tables. Every slot of every (N-block, K-chunk) holds exactly c inputs with signs
 * +-1, so the projection is the sketch of each weight row, divided by c:
 *
 *     Wc[n, j] = (1 / c) * sum over k with h_nb(k) == j of g_nb(k) * W[n, k],   nb = n / BN.
 *
 * Projecting a tied weight (W = W_full(Wc0)) returns Wc0 exactly.
 *   W     : device, [N, K] of `dtype` (torch.nn.Linear layout: one row per output neuron).
 *   Wc    : device, [N, K / c] of `dtype`, written in full; must not overlap W.
 *   dtype : SS1_DTYPE_BF16 or SS1_DTYPE_FP32; the c terms are summed in fp32 and rounded once.
 *   stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 * The caller owns W and Wc. Asynchronous; reads the handle only, so calls may run concurrently.
 * Rows and K-chunks of W that are multiples of 16 bytes, with W 16-byte aligned, take the fast
 * kernels (rows streamed through shared memory; bf16 rows in pairs); any other shape a plain
 * one. Errors: BAD_HANDLE, INVALID_ARG (NULL pointer, dtype),
 * MISALIGNED (W or Wc not aligned to its element size), CUDA (launch failure).
 */
SS1_API int ss1_project(ss1_handle h, const void* W, void* Wc, int dtype, void* stream);

/*
 * Backward pass. "SS1: Accelerating Inference with Fast and Expressive Sketch Structured
 * Transform", section "Limitations": SS1 does not make the backward pass cheaper. The pages give
 * no formula; on the tied weight W_full[n, k] = g_nb(k) Wc[n, h_nb(k)] matrix calculus gives, for
 * dY = dLoss/dY [M, N],
 *
 *     dX[m, k]  = sum_n dY[m, n] W_full[n, k]                                     [M, K]
 *     dWc[n, j] = sum over k with h_nb(k) == j of g_nb(k) * sum_m dY[m, n] X[m, k]   [N, K / c]
 *
 * Both run at the dense layer's cost (as the pages describe): W_full^T, or dY^T and X^T, are
 * written into a caller-provided workspace and multiplied on the tensor cores (bf16 shapes with
 * K a multiple of 128 and, for dX, N a multiple of 64) or the CUDA cores (fp32, other shapes),
 * accumulating in fp32. The workspace is device memory of at least the size that
 * ss1_backward_workspace gives, 256-byte aligned, owned by the caller, not read before it is
 * written; calls that share one workspace must be ordered on the device. Both calls are
 * asynchronous and only read the handle.
 */

/*
 * ss1_backward_workspace -- workspace bytes of ss1_backward_input (independent of M) and of
 * ss1_backward_weight for M rows; either output pointer may be NULL. Errors: BAD_HANDLE,
 * INVALID_ARG (M < 0, dtype).
 */
SS1_API int ss1_backward_workspace(ss1_handle h, int64_t M, int dtype, size_t* input_bytes, size_t* weight_bytes);

/*
 * ss1_backward_input -- dX = dY W_full.
 *   dY : device, [M, N] of `dtype`.     Wc : device, [N, K / c].     dX : device, [M, K], written.
 *   workspace, workspace_bytes : see above (W_full^T, K * N elements).
 * M == 0 is a no-op. Errors: BAD_HANDLE, INVALID_ARG (sizes, dtype, NULL pointer, workspace too
 * small), MISALIGNED (dY, Wc, dX not 16-byte or workspace not 256-byte aligned), CUDA,
 * DEVICE_TIMEOUT (as for ss1_forward).
 */
SS1_API int ss1_backward_input(ss1_handle h, const void* dY, const void* Wc, void* dX, int64_t M, int dtype,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * ss1_backward_weight -- dWc, the gradient with respect to the compressed weights.
 *   X  : device, [M, K] of `dtype` (the forward's input).   dY : device, [M, N].
 *   dWc: device, [N, K / c], written (overwritten, not accumulated); zero when M == 0.
 *   workspace, workspace_bytes : see above (dY^T and X^T padded to a multiple of 64 rows, and
 *   the dense gradient dY^T X).
 * Errors: as ss1_backward_input (X, dY, dWc 16-byte aligned).
 */
SS1_API int ss1_backward_weight(ss1_handle h, const void* X, const void* dY, void* dWc, int64_t M, int dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * FP8 weights. "SS1: Accelerating Inference with Fast and Expressive Sketch Structured
 * Transform", section "Limitations": quantised SS1 kernels were not built; section "Measured
 * effects": post-training quantisation of SS1 models. The pages fix no format; this library
 * stores the compressed weights as OCP FP8 E4M3 codes (1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits, largest magnitude 448, no infinities) with one float scale per output neuron:
 *
 *     Wc_deq[n, j] = scale[n] * e4m3(Wq[n, j]),   Y = SS1(X) computed with Wc_deq.
 */

/*
 * ss1_quantize_fp8 -- per-neuron FP8 quantisation of compressed weights (no handle needed).
 *   Wc    : device, [N, Kc] of `dtype` (bf16 or fp32).
 *   Wq    : device, [N, Kc] bytes, written: E4M3 codes of Wc[n, j] / scale[n], rounded to nearest
 *           even, magnitudes past 448 saturated to 448.
 *   scale : device, [N] float, written: max_j |Wc[n, j]| / 448 (correctly rounded float32
 *           division), or 1 for an all-zero row.
 * Asynchronous. Errors: INVALID_ARG (sizes, dtype, NULL), MISALIGNED (Wc not aligned to its
 * element, scale to 4 bytes), CUDA.
 */
SS1_API int ss1_quantize_fp8(const void* Wc, int dtype, int64_t N, int64_t Kc, void* Wq, float* scale, void* stream);

/*
 * ss1_forward_fp8 -- Y = SS1(X) with FP8 weights (Wq, scale), for decode-sized batches.
 *   X : device, bf16 [M, K].   Wq : device, [N, K / c] E4M3 codes.   scale : device, float [N].
 *   Y : device, bf16 [M, N], written.   M : 0 .. 64 (M == 0 is a no-op).
 * Runs the tensor-core decode kernel: Wc streams as one byte per weight, each stage is widened
 * to bf16 on chip (exactly), the sketch is as in ss1_forward, products accumulate in fp32, and
 * Y[m, n] = bf16(scale[n] * sum). Re-entrant like ss1_forward.
 * Errors: BAD_HANDLE, INVALID_ARG, MISALIGNED (X, Wq, Y 16-byte, scale 4-byte aligned),
 * UNSUPPORTED_SHAPE (M > 64, BN != 128, K / c not a multiple of 16), CUDA, DEVICE_TIMEOUT.
 */
SS1_API int ss1_forward_fp8(ss1_handle h, const void* X, const void* Wq, const float* scale, void* Y, int64_t M,
                            void* stream);

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
 * padding), then runs the kernel ss1_forward would choose, with the same results bit for bit.
 * Shapes with (N / BN) * K > SS1_NOALLOC_MAX_ENTRIES are rejected with UNSUPPORTED_SHAPE. No
 * cudaMalloc, cudaFree, pinned allocation or allocating library routine is called, and
 * nothing synchronises the device; the tables need no zeroing because the table kernels
 * write all of them that the forward reads.
 *
 * The first call on a device does one-time set-up (it looks up the region's address and
 * sets kernel attributes); make that first call outside any stream capture. The set-up belongs
 * to the device's CUDA context: after cudaDeviceReset the next call on that device runs it
 * again in the new context (so that call, too, should come before any stream capture).
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

/*
 * ss1_test_forward_timeout -- exercises a forward kernel's own time-out path without a fault, for
 * tests of failure handling (the SS1 pages have no counterpart). Runs the tensor-core kernel for
 * c >= 2 (the one ss1_forward picks for large bf16 batches) on X, Wc, Y as ss1_forward would
 * (a test variant of it, built for layers with BK = 128, c = 2 and an even count of N-blocks),
 * with every bounded wait cut to limit_ns nanoseconds (1 .. 2e9) and CTA 0's first sketch-matrix
 * warp withholding its arrival for the third sketch segment, so CTA 0 stalls. The first of its
 * waits to run out writes the status word ((1 << 8) | 0x80 | site: kernel id 1, the wait's site),
 * the CTA's other warps give up their waits, every copy and matrix multiply in flight completes,
 * the tensor memory is freed and the kernel returns; Y is not valid. Afterwards ss1_forward on this handle
 * returns SS1_ERR_DEVICE_TIMEOUT until ss1_device_status has read and cleared the word.
 * Asynchronous. Errors: BAD_HANDLE, INVALID_ARG (limit_ns out of range, M < 1, NULL pointer),
 * MISALIGNED, UNSUPPORTED_SHAPE (not such a layer), CUDA.
 */
SS1_API int ss1_test_forward_timeout(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M, int64_t limit_ns,
                                     void* stream);

/*
 * ss1_last_launch -- the shape of the main kernel that the last layer entry point (ss1_forward,
 * _with, _ex, ss1_chain_forward, ss1_forward_fp8, ss1_forward_noalloc) called on this host thread
 * launched: which kernel, its grid, cluster and block. For checking that a launch uses the
 * machine as intended (how many CTAs, how K is split); it has no counterpart on the SS1 pages.
 *   kernel : static name: "tc3" (large-M tensor-core kernel, c >= 2), "tc" (c = 1; a grid of
 *            at most one CTA per SM where N is a multiple of 256 and M is large), "tc2",
 *            "simt", "dec" (tensor-core decode kernel), "dec_fp8", "smallm"; "" before any launch.
 *   grid_x, grid_y : CTAs of the grid (grid_y: K-splits where the kernel splits K).
 *   cluster_y : CTAs per thread-block cluster along y (1: no cluster).
 *   threads, smem_bytes : per CTA (dynamic shared memory).
 *   resident_clusters[s], s = 1 .. 16 : what the occupancy query behind the K-split choice
 *            reported (clusters of s CTAs resident at once); all 0 where none was made.
 * out : host pointer. Errors: INVALID_ARG (NULL).
 */
typedef struct {
    const char* kernel;
    int grid_x, grid_y;
    int cluster_y;
    int threads;
    int smem_bytes;
    int resident_clusters[17];
} ss1_launch_info;
SS1_API int ss1_last_launch(ss1_launch_info* out);

/*
 * ss1_bounds_check -- the record of the checked (debug) build, libss1_checked.so: the same
 * sources compiled so that every global-memory access a kernel addresses by its own index
 * arithmetic first tests its element index against the extent of the buffer (tables, X, Wc, Y,
 * scales, bias, the backward and projection operands). A failed test skips the access and
 * records the first failure; TMA tile copies are bounded by their tensor maps in hardware. The
 * normal build makes no tests and has the same entry point.
 *   checked : receives 1 in the checked build, 0 in the normal one.
 *   record  : receives the first failed test on the current device since the last call, 0 if
 *             none: (site << 48) | (element index mod 2^48), site a small positive number
 *             naming the access; the record is then cleared. Always 0 in the normal build.
 * The checked build synchronises the current device first (no other effect on the caller's
 * work). Host pointers. Errors: INVALID_ARG (NULL), CUDA (checked build only).
 */
SS1_API int ss1_bounds_check(int* checked, uint64_t* record);

/*
 * ss1_test_bounds_check -- the checked build's index test run once on the given values, for
 * tests of the record itself: one thread on the legacy default stream of the current device
 * tests `index` against `extent` elements (site 63) and accesses no memory. When the index is
 * out of range, the next ss1_bounds_check reports (63 << 48) | index. Asynchronous.
 * Errors: UNSUPPORTED_SHAPE in the normal build (nothing is launched), CUDA.
 */
SS1_API int ss1_test_bounds_check(int64_t index, int64_t extent);

#ifdef __cplusplus
}
#endif

#endif /* SS1_H */
