// Tensor-core SS1 forward for decode-sized batches (M <= 64 rows, bf16, N-blocks of 128).
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": the input is sketched (signed hashed additions shrink each K-chunk by c) and the
// sketch is multiplied with the compressed weights. With a few rows the product is bound by
// reading Wc (N x K/c bf16) once. Here the 128 neurons of an N-block are the UMMA's M:
//
//     D[n, m] += Wc[n, j] * Xs_nb[m, j]      (A = Wc, streamed by TMA; B = the rows' sketch)
//
// with UMMA N = the row count rounded up to 16, so the tensor pipe is busy a few percent of the
// time and the kernel is a TMA stream of Wc.
//
// CTA = (N-block nb, K-split s): the split's stages of 64 compressed columns; one CTA per SM.
//   warp 0     : lane 0 copies the CTA's X columns (one bulk copy per row) where they fit in
//                shared memory, then refills a ring of Wc stages [128 neurons x 64 columns]
//                (128-byte swizzle; bf16 8 x 16 KB, FP8 22 x 8 KB) by TMA in stage order.
//   warp 1     : TMEM allocation; lane 0 issues 4 UMMAs (K = 16) per stage for the even stages
//                (bf16; FP8 every stage); warp 6 (bf16) the odd stages into a second
//                accumulator; the epilogue adds the two in order.
//   warps 2..5 : the sketch of each stage, Xs[m, j] = sum_t sign_t * X[m, chunk(j) * BK + k_t]
//                (fp32 sum, one rounding to bf16), into a swizzled B stage (warps 2-3 the even
//                stages, warps 4-5 the odd ones), gathering from shared memory: the CTA's X
//                columns copied in once; or, for up to 16 rows whose columns do not fit, the X
//                rows of each unit (one K-chunk of whole stages, or one stage of whole K-chunks)
//                by TMA (one more lane of warp 0) into a ring of up to eight units; else the
//                gathers go to L1 / L2. Then the epilogue.
// Before the dependency wait of a programmatic dependent launch the CTA asks L2 for its X
// columns and its first Wc stages.
// Epilogue: TMEM -> D[n, m]. One split: Y[m, n] = bf16(D[n, m]). Several: the K-splits of one
// N-block form one thread-block cluster. Every CTA leaves its fp32 partial [rows x 128 neurons]
// in its own shared memory; after a cluster barrier, CTA r sums rows r, r + splits, ... over the
// splits' partials, read through distributed shared memory in split order (the same bits every
// call), and writes them to Y. Nothing is written outside X, Wc and Y, so calls are re-entrant.
// Every mbarrier wait is bounded; a wait that runs out sets the CTA's abort flag and the status
// word, and every thread still reaches both cluster barriers.
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace ss1 {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

constexpr int kNeu = 128;                 // neurons per N-block = UMMA M
constexpr int kStageC = 64;               // compressed columns per stage (one 128-byte swizzle row)
constexpr int kWRingFp8 = 176 * 1024;     // shared memory of the FP8 Wc ring: 22 stages
constexpr int kNwBf16 = 8;                // bf16 Wc stages in the ring
constexpr int kNmmaBf16 = 2;              // bf16 UMMA warps
constexpr int kXBytes = 20 * 1024;       // X in shared memory: the CTA's input range, or the chunk ring
constexpr int kXChunkRows = 16;          // chunk mode: rows of an X box (M <= 16)
constexpr int kXUnitBytes = kXChunkRows * 512 * 2;    // one unit: [16 rows x up to 512 inputs]
constexpr int kMaxXUnits = 8;             // chunk mode: X units in flight at most
// Build warps from kFirstBuild: bf16, two row parts of kEpiWarps warps; FP8, one part (the
// converter warps come after them). The first part also runs the epilogue.
constexpr int kWarpLoad = 0, kWarpMma = 1, kFirstBuild = 2, kEpiWarps = 4, kConvWarps = 4;
constexpr uint64_t kWaitNs = 2000000000ull;

// L2 prefetch of one 2D tile of a tensor map: no shared memory, no completion to wait for.
// c0 * 2 bytes must be a multiple of 16, as for a tiled load.
__device__ __forceinline__ void prefetch_l2_2d(const CUtensorMap* map, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

// L2 prefetch of a contiguous range (16-byte aligned, a multiple of 16 bytes).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes) : "memory");
}

// Programmatic dependent launch. pdl_wait blocks until the grids this one depends on have
// completed and their memory is visible; for a launch without the attribute it returns at once.
// pdl_launch_dependents lets a dependent grid be scheduled once every CTA of this grid has
// issued it or exited (the dependent still waits for this grid's completion in pdl_wait).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// FP8 = true: Wc arrives as E4M3 codes [128 neurons x 64 columns] (8 KB, 64-byte swizzle); four
// converter warps widen each stage to bf16 (exact) straight into TMEM, where it is the UMMA's A
// operand, and the epilogue multiplies neuron n's sum by its scale.
template <int MP, bool FP8>
struct DecCfg {
    static constexpr int W_STAGE = kNeu * kStageC * (FP8 ? 1 : 2);   // 8 or 16 KB
    static constexpr int NW = FP8 ? kWRingFp8 / W_STAGE : kNwBf16;   // Wc stages in the ring
    // bf16: NMMA UMMA warps take the stages round-robin into NMMA accumulators, so that the
    // barrier waits of one (each lets the tensor pipe's queue drain) overlap the others' UMMAs
    static constexpr int NMMA = FP8 ? 1 : kNmmaBf16;
    static constexpr int ROW_PARTS = FP8 ? 1 : 2;
    static constexpr int BUILD_WARPS = kEpiWarps * ROW_PARTS;
    static constexpr int FIRST_CONV = kFirstBuild + BUILD_WARPS;   // FP8: the converter warps, from here
    static constexpr int WARP_MMA2 = kFirstBuild + BUILD_WARPS;    // bf16: the further UMMA warps, from here
    static constexpr int THREADS = (kFirstBuild + BUILD_WARPS + (FP8 ? kConvWarps : NMMA - 1)) * 32;
    // one CTA per SM with a deep ring: a stage stays in the ring from its load until its UMMAs
    // complete, and about 128 KB per SM must be on the way from HBM at any time for it to run at
    // its rate at the latency it has under that load
    static constexpr int MIN_CTAS = 1;
    static constexpr int B_STAGE = MP * 128;                    // [MP rows x 64] bf16
    // sketch stages in the ring (the build warps run ahead of the UMMAs); FP8 three, each also
    // holding a bf16 A stage in TMEM
    static constexpr int NBS = FP8 ? 3 : 4;
    static constexpr int OFF_W = 0;
    static constexpr int OFF_B = NW * W_STAGE;
    static constexpr int OFF_X = OFF_B + NBS * B_STAGE;
    // X: for up to 16 rows the ring of units (or the CTA's range), else the range
    static constexpr int X_BYTES = MP == kXChunkRows ? (FP8 ? 2 * kXUnitBytes : 80 * 1024) : kXBytes;
    static constexpr int OFF_BAR = OFF_X + X_BYTES;
    static constexpr int NBAR = 2 * NW + 2 * NBS + 1 + 2 * kMaxXUnits;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    // accumulator MP columns; FP8: plus NBS bf16 A stages of 32 columns from A_COL
    static constexpr int A_COL = MP <= 32 ? 32 : 64;
    static constexpr uint32_t TMEM_COLS = FP8 ? (MP <= 32 ? 128 : 256) : (uint32_t)(NMMA * MP < 32 ? 32 : NMMA * MP);
    static_assert(MP % 16 == 0 && MP >= 16 && MP <= 64, "UMMA N for M = 128");
    static_assert(B_STAGE % 1024 == 0 && OFF_B % 1024 == 0, "swizzle atoms stay aligned");
    static_assert(!FP8 || (A_COL >= MP && A_COL + NBS * 32 <= (int)TMEM_COLS), "TMEM layout");
    static_assert(NW <= 31, "the chunk-mode X loader is lane NW of the load warp");
    static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
    // a ring slot's successive uses go to one UMMA warp, which waits for them in order (a wait on
    // a barrier's phase parity must never be able to see the phase two uses back)
    static_assert(NW % NMMA == 0 && NBS % NMMA == 0, "ring depths are multiples of the UMMA warps");
};

// Two E4M3 codes (low byte = the even column) -> bf16x2, exactly: every E4M3 value has at most
// four significant bits and an exponent inside bf16's range.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ void report(int32_t* status, volatile int* abort_flag, int site) {
    *abort_flag = 1;
    *(volatile int32_t*)status = (kStatusKernelDec << 8) | (0x80 + site);
    __threadfence_system();
}

// Lane 0 waits, the warp follows.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, abort_flag, kWaitNs);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Wait of the UMMA-issuing warp: every lane polls without suspending, so the issue resumes as
// soon as the phase completes (a suspending wait costs the issuing thread several hundred cycles).
__device__ __forceinline__ bool warp_wait_spin(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
    bool ok = ptx::mbar_test(bar, parity);
    if (!ok) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (uint32_t n = 1;; ++n) {
            if (ptx::mbar_test(bar, parity)) { ok = true; break; }
            if ((n & 63) == 0 && (*abort_flag || ptx::globaltimer_ns() - t0 > kWaitNs)) break;
        }
    }
    return __all_sync(0xffffffffu, ok);
}

template <int MP, int C, bool FP8>
__global__ void __launch_bounds__(DecCfg<MP, FP8>::THREADS, DecCfg<MP, FP8>::MIN_CTAS)
    dec_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
               const __nv_bfloat16* __restrict__ X, __nv_bfloat16* __restrict__ Y, const uint16_t* __restrict__ src,
               const float* __restrict__ scale, int M, int K, int N, int S, int KC, int splits, int chunked, int ui,
               int bi, int32_t* status) {
    using F = DecCfg<MP, FP8>;
    constexpr int kNW = F::NW, kWStage = F::W_STAGE, kThreads = F::THREADS, kACol = F::A_COL, kNB = F::NBS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* wring = smem + F::OFF_W;
    uint8_t* bring = smem + F::OFF_B;
    uint64_t* w_full = reinterpret_cast<uint64_t*>(smem + F::OFF_BAR);
    uint64_t* w_empty = w_full + kNW;
    uint64_t* b_full = w_empty + kNW;     // the two build warps (and, FP8, the four converter warps) are done
    uint64_t* b_empty = b_full + kNB;     // the stage's UMMAs have completed (its B stage and A stage are free)
    uint64_t* acc_full = b_empty + kNB;
    uint64_t* x_full = acc_full + 1;      // [kMaxXUnits] chunk mode: an X unit has landed
    uint64_t* x_empty = x_full + kMaxXUnits;   // [kMaxXUnits] chunk mode: every stage of the unit has been built
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_empty + kMaxXUnits);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nb = blockIdx.x, split = blockIdx.y;
    const int Kc = K / C;
    const int nstg = (Kc + kStageC - 1) / kStageC;
    // Stages [st0, st1) of this CTA. Chunk mode (M <= 16): whole units, a unit being the X
    // inputs of one K-chunk of S / 64 stages (S a multiple of 64) or of one stage spanning
    // 64 / S chunks; so every unit a CTA touches is one it uses entirely. ui = inputs per unit
    // (contiguous in X), bi = inputs per TMA box (ui or 256).
    const int spc = chunked ? (S >= kStageC ? S / kStageC : 1) : 1;   // stages per unit
    int st0, st1;
    if (chunked) {
        const int nu = S >= kStageC ? KC : nstg;
        st0 = (int)((int64_t)nu * split / splits) * spc;
        st1 = (int)((int64_t)nu * (split + 1) / splits) * spc;
    } else {
        st0 = (int)((int64_t)nstg * split / splits);
        st1 = (int)((int64_t)nstg * (split + 1) / splits);
    }
    const int G = st1 - st0;   // stages of this CTA (>= 1)
    // Outside chunk mode the X columns of this CTA's K-chunks (all rows) are copied into shared
    // memory once where they fit (one bulk copy per row; then every gather is a shared-memory
    // read); else the gathers go to L1 / L2.
    const int BKc = S * C;
    const int kc_lo = (st0 * kStageC) / S;
    const int kc_hi = (min(st1 * kStageC, Kc) - 1) / S;
    const int R = (kc_hi - kc_lo + 1) * BKc;   // inputs of the range
    const bool staged = !chunked && BKc % 8 == 0 && (int64_t)M * R * 2 <= F::X_BYTES;   // 16-byte aligned rows
    // chunk mode: X units [16 rows x ui] in flight, as many as the X region holds (at most kMaxXUnits)
    const int xub = kXChunkRows * ui * 2;
    const int nxu = chunked ? min(kMaxXUnits, F::X_BYTES / xub) : 1;

    // row parts of the build (bf16): the second (rows MP / 2 ..) only where M reaches it
    const int nrp = F::ROW_PARTS == 2 && M > MP / 2 ? 2 : 1;

    // sketch stages start zeroed: rows past M are never written afterwards
    for (int i = threadIdx.x; i < kNB * F::B_STAGE / 16; i += kThreads)
        reinterpret_cast<uint4*>(bring)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        // FP8: a Wc slot is free once the converter warps have read it (bf16: once its UMMAs completed)
        for (int i = 0; i < kNW; ++i) { ptx::mbar_init(&w_full[i], 1); ptx::mbar_init(&w_empty[i], FP8 ? kConvWarps : 1); }
        for (int i = 0; i < kNB; ++i) {
            ptx::mbar_init(&b_full[i], kEpiWarps / 2 * nrp + (FP8 ? kConvWarps : 0));
            ptx::mbar_init(&b_empty[i], 1);
        }
        ptx::mbar_init(acc_full, F::NMMA);
        for (int i = 0; i < kMaxXUnits; ++i) {
            ptx::mbar_init(&x_full[i], 1);
            ptx::mbar_init(&x_empty[i], kEpiWarps / 2 * nrp * (chunked ? spc : 1));
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(tmem_slot, F::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == kWarpLoad && lane == 0) ptx::prefetch_tmap(&tmap_w);
    if (warp == kWarpLoad && lane == kNW && chunked) ptx::prefetch_tmap(&tmap_x);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tm = *tmem_slot;

    // The launch may overlap the end of the previous kernel on the stream (programmatic
    // dependent launch). Until that kernel has completed, this CTA only asks L2 for its X columns
    // and the first Wc stages it will stream: a prefetch goes through L2, so it cannot return
    // data older than what that kernel writes. Every global read and write below comes after
    // the wait.
    if (warp == kWarpLoad && lane == 0) {
        if (staged)
            for (int m = 0; m < M; ++m)
                if (SS1_SPAN_IN((size_t)m * K + (size_t)kc_lo * BKc, R, (int64_t)M * K, kSiteDecX))
                    prefetch_l2_bulk(X + (size_t)m * K + (size_t)kc_lo * BKc, (uint32_t)(R * 2));
        for (int g = 0; g < G && g < kNW; ++g)
            prefetch_l2_2d(&tmap_w, (st0 + g) * kStageC, nb * kNeu);
    }
    if (threadIdx.x == 0) pdl_launch_dependents();
    pdl_wait();

    if (warp == kWarpLoad) {
        // ------------------------------------------------------------------ TMA loads
        // The X columns first (the sketch waits for them), one bulk copy per row, by lane 0.
        if (staged && lane == 0) {
            ptx::mbar_arrive_expect_tx(&x_full[0], (uint32_t)(M * R * 2));
            for (int m = 0; m < M; ++m)
                if (SS1_SPAN_IN((size_t)m * K + (size_t)kc_lo * BKc, R, (int64_t)M * K, kSiteDecX))
                    ptx::bulk_load(smem + F::OFF_X + (size_t)m * R * 2, X + (size_t)m * K + (size_t)kc_lo * BKc,
                                   (uint32_t)(R * 2), &x_full[0]);
        }
        __syncwarp();
        // Wc: lane 0 refills the ring in stage order (stage g into slot g % kNW once the UMMAs of
        // stage g - kNW have completed). Issuing from several lanes was measured no faster: the
        // copies of one SM are served one after another either way.
        if (lane == 0) {
            int issued = 0;
            for (int g = 0; g < G; ++g) {
                const int slot = g % kNW;
                if (g >= kNW && !ptx::mbar_wait(&w_empty[slot], (uint32_t)(((g / kNW) - 1) & 1), abort_flag, kWaitNs)) {
                    report(status, abort_flag, 1);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&w_full[slot], kWStage);
                ptx::tma_load_2d(wring + slot * kWStage, &tmap_w, &w_full[slot], (st0 + g) * kStageC, nb * kNeu);
                ++issued;
            }
            if (*abort_flag) {   // the copies in flight land before exit
                volatile int no_abort = 0;
                for (int g = issued > kNW ? issued - kNW : 0; g < issued; ++g)
                    ptx::mbar_wait(&w_full[g % kNW], (uint32_t)((g / kNW) & 1), &no_abort, kWaitNs);
            }
        } else if (lane == kNW && chunked) {
            // X units [16 rows x ui] (rows past M read as zero) into a ring of nxu, as boxes of
            // [16 x bi] stored one after another
            const int nun = G / spc, un0 = st0 / spc;
            int issued = 0;
            for (int u = 0; u < nun; ++u) {
                const int xs = u % nxu;
                if (u >= nxu && !ptx::mbar_wait(&x_empty[xs], (uint32_t)(((u / nxu) - 1) & 1), abort_flag, kWaitNs)) {
                    report(status, abort_flag, 5);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&x_full[xs], (uint32_t)xub);
                for (int b = 0; b < ui / bi; ++b)
                    ptx::tma_load_2d(smem + F::OFF_X + xs * xub + b * (kXChunkRows * bi * 2), &tmap_x,
                                     &x_full[xs], (un0 + u) * ui + b * bi, 0);
                ++issued;
            }
            if (*abort_flag) {
                volatile int no_abort = 0;
                for (int u = issued > nxu ? issued - nxu : 0; u < issued; ++u)
                    ptx::mbar_wait(&x_full[u % nxu], (uint32_t)((u / nxu) & 1), &no_abort, kWaitNs);
            }
        }
        if (staged && lane == 0 && *abort_flag) {   // the X copies land before exit
            volatile int no_abort = 0;
            ptx::mbar_wait(&x_full[0], 0, &no_abort, kWaitNs);
        }
    } else if (warp == kWarpMma || (F::NMMA > 1 && warp >= F::WARP_MMA2 && warp < F::WARP_MMA2 + F::NMMA - 1)) {
        // ------------------------------------------------------------------ UMMAs
        // UMMA warp w (w < NMMA) takes stages g = w, w + NMMA, ... into accumulator w (MP columns
        // from w * MP).
        const int w = warp == kWarpMma ? 0 : warp - F::WARP_MMA2 + 1;
        const uint32_t dacc = tm + (uint32_t)(w * MP);
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(kNeu, MP);
        const uint64_t wdesc0 = ptx::smem_desc(ptx::smem_u32(wring), 16, 1024, ptx::kLayoutSW128);
        const uint64_t bdesc0 = ptx::smem_desc(ptx::smem_u32(bring), 16, 1024, ptx::kLayoutSW128);
        bool ok = true;
        for (int g = w; g < G && ok; g += F::NMMA) {
            const int ws_ = g % kNW, bs = g % kNB;
            if ((!FP8 && !warp_wait_spin(&w_full[ws_], (uint32_t)((g / kNW) & 1), abort_flag)) ||
                !warp_wait_spin(&b_full[bs], (uint32_t)((g / kNB) & 1), abort_flag)) {
                if (lane == 0) report(status, abort_flag, 2);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            if (lane == 0) {
                const uint64_t wd = wdesc0 + (uint64_t)((ws_ * kWStage) >> 4);
                const uint64_t bd = bdesc0 + (uint64_t)((bs * F::B_STAGE) >> 4);
                const uint32_t at = tm + (uint32_t)(kACol + bs * 32);   // FP8: the stage's bf16 A in TMEM
#pragma unroll
                for (int kk = 0; kk < kStageC / 16; ++kk) {
                    if (FP8)
                        ptx::umma_bf16_ts(dacc, at + (uint32_t)(kk * 8), bd + (uint64_t)(kk * 2), idesc, (g > w || kk > 0) ? 1u : 0u);
                    else
                        ptx::umma_bf16_ss(dacc, wd + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (g > w || kk > 0) ? 1u : 0u);
                }
                if (!FP8 && g + kNW < G) ptx::umma_commit(&w_empty[ws_]);   // only a slot used again
                if (g + kNB < G) ptx::umma_commit(&b_empty[bs]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            ptx::umma_commit(acc_full);
            if (*abort_flag) {   // the UMMAs in flight finish before TMEM is released
                volatile int no_abort = 0;
                ptx::mbar_wait(acc_full, 0, &no_abort, kWaitNs);
            }
        }
        __syncwarp();
    } else if (FP8 && warp >= F::FIRST_CONV) {
        // ------------------------------------------------------------------ FP8 -> bf16 A stages
        // Thread = neuron (TMEM lane 32 q + lane, q = warp % 4): its row of the stage, 64 codes in
        // four 16-byte chunks (64-byte swizzle: chunk c of row r sits at c ^ ((r >> 1) & 3), so
        // eight rows read per wavefront hit distinct banks), widened to 32 bf16x2 words and
        // stored into the stage's TMEM columns.
        const int q = warp & 3, r = q * 32 + lane;
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        bool ok = true;
        for (int g = 0; g < G && ok; ++g) {
            const int ws_ = g % kNW, bs = g % kNB;
            if (!warp_wait(&w_full[ws_], (uint32_t)((g / kNW) & 1), abort_flag) ||
                (g >= kNB && !warp_wait(&b_empty[bs], (uint32_t)(((g / kNB) - 1) & 1), abort_flag))) {
                if (lane == 0) report(status, abort_flag, 7);
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint8_t* row = wring + ws_ * kWStage + r * 64;
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 u = *reinterpret_cast<const uint4*>(row + ((c ^ ((r >> 1) & 3)) << 4));
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[c * 8 + 2 * e] = e4m3x2_to_bf16x2((uint16_t)(w4[e] & 0xFFFFu));
                    v[c * 8 + 2 * e + 1] = e4m3x2_to_bf16x2((uint16_t)(w4[e] >> 16));
                }
            }
            ptx::tmem_st_32x32b_x16(tm + lanes + (uint32_t)(kACol + bs * 32), *reinterpret_cast<const uint32_t(*)[16]>(v));
            ptx::tmem_st_32x32b_x16(tm + lanes + (uint32_t)(kACol + bs * 32 + 16), *reinterpret_cast<const uint32_t(*)[16]>(v + 16));
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&w_empty[ws_]);   // the codes have been read
                ptx::mbar_arrive(&b_full[bs]);     // the A stage is in TMEM
            }
        }
    } else {
        // ------------------------------------------------------------------ sketch, then epilogue
        // Build thread t: column kl = t % 64 of the stages g with g % 2 == (t / 64) % 2 (two stages
        // are built at once), the rows of row part rp = t / 128 (bf16: rows 0 .. MP / 2 - 1 and
        // MP / 2 .., FP8: all). A thread's table entries are loaded one of its stages ahead, so
        // that a stage waits only for its X gathers, which are all in flight together. A second
        // row part builds only where M reaches it; the first also runs the epilogue.
        constexpr int kRowsPart = MP / F::ROW_PARTS;
        const int t = threadIdx.x - kFirstBuild * 32;
        const int kl = t % kStageC, half = (t / kStageC) & 1, rp = t / (2 * kStageC);
        const bool builds = rp < nrp;
        const int BK = BKc;
        const uint16_t* tab = src + (size_t)nb * KC * S * C;   // this N-block's entries, column-major order
        auto fetch = [&](int g, uint16_t (&e)[C]) {
            const int j = (st0 + g) * kStageC + kl;
            if (g < G && j < Kc) {
#pragma unroll
                for (int q = 0; q < C; ++q)
                    e[q] = SS1_IN(tab + (size_t)j * C + q - src, (int64_t)(N / kNeu) * K, kSiteDecTab)
                               ? __ldg(tab + (size_t)j * C + q)
                               : (uint16_t)0;
            }
        };
        const __nv_bfloat16* xsm = reinterpret_cast<const __nv_bfloat16*>(smem + F::OFF_X);
        uint16_t ent[C];
        fetch(half, ent);   // in flight together with the X copy
        bool ok = true;
        if (staged && !warp_wait(&x_full[0], 0, abort_flag)) {   // the CTA's X columns have landed
            if (lane == 0) report(status, abort_flag, 8);
            ok = false;
        }
        for (int g = half; g < G && ok && builds; g += 2) {
            const int bs = g % kNB;
            uint16_t cur[C];
#pragma unroll
            for (int q = 0; q < C; ++q) cur[q] = ent[q];
            fetch(g + 2, ent);
            if (g >= kNB && !warp_wait(&b_empty[bs], (uint32_t)(((g / kNB) - 1) & 1), abort_flag)) {
                if (lane == 0) report(status, abort_flag, 3);
                ok = false;
                break;
            }
            uint8_t* stage = bring + bs * F::B_STAGE;
            const int j = (st0 + g) * kStageC + kl;   // compressed column
            const int u = chunked ? g / spc : 0;      // chunk mode: the stage's unit in this CTA
            if (chunked && !warp_wait(&x_full[u % nxu], (uint32_t)((u / nxu) & 1), abort_flag)) {
                if (lane == 0) report(status, abort_flag, 6);
                ok = false;
                break;
            }
            if (j < Kc) {
                const int kc = j / S;   // the column's K-chunk
                // chunk mode: the chunk's inputs start at ii0 within its unit, inside one box
                const int ii0 = chunked ? kc * BK - (st0 / spc + u) * ui : 0;
                const __nv_bfloat16* xk = chunked  ? xsm + (size_t)(u % nxu) * (xub / 2) +
                                                         (size_t)(ii0 / bi) * (kXChunkRows * bi) + (ii0 % bi)
                                          : staged ? xsm + (size_t)(kc - kc_lo) * BK
                                                   : X + (size_t)kc * BK;
                const size_t row = chunked ? (size_t)bi : staged ? (size_t)R : (size_t)K;
#pragma unroll(kRowsPart > 16 ? 16 : kRowsPart)
                for (int mi = 0; mi < kRowsPart; ++mi) {
                    const int m = rp * kRowsPart + mi;
                    if (m < M) {
                        float v = 0.f;
#pragma unroll
                        for (int q = 0; q < C; ++q) {
                            const size_t xi = (size_t)m * row + (cur[q] & kSrcIdxMask);
                            const float x = (chunked || staged || SS1_IN(xk + xi - X, (int64_t)M * K, kSiteDecX))
                                                ? __bfloat162float(xk[xi])
                                                : 0.f;
                            v += (cur[q] & kSrcNegBit) ? -x : x;
                        }
                        *reinterpret_cast<__nv_bfloat16*>(stage + m * 128 + (((kl >> 3) ^ (m & 7)) << 4) + (kl & 7) * 2) =
                            __float2bfloat16_rn(v);
                    }
                }
            } else {
#pragma unroll
                for (int mi = 0; mi < kRowsPart; ++mi) {
                    const int m = rp * kRowsPart + mi;
                    if (m < M)
                        *reinterpret_cast<uint16_t*>(stage + m * 128 + (((kl >> 3) ^ (m & 7)) << 4) + (kl & 7) * 2) = 0;
                }
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&b_full[bs]);
                if (chunked) ptx::mbar_arrive(&x_empty[u % nxu]);   // this stage's reads of the unit are done
            }
        }
        // epilogue: warp (quad) holds neurons nb * 128 + quad * 32 + lane
        const int quad = warp & 3;
        if (rp > 0) {
            // the second row part holds no accumulator lanes of its own
        } else if (ok && warp_wait(acc_full, 0, abort_flag) && !*abort_flag) {
            ptx::tc_fence_after();
            const int n = nb * kNeu + quad * 32 + lane;
            const float sc = FP8 && splits == 1 && SS1_IN(n, N, kSiteDecScale) ? scale[n] : 1.0f;
            // this split's partial [MP rows][128 neurons] fp32 goes into the Wc ring: every stage
            // has been multiplied (acc_full), so the ring is free
            float* part = reinterpret_cast<float*>(wring) + quad * 32 + lane;
#pragma unroll
            for (int m0 = 0; m0 < MP; m0 += 16) {   // 16 rows at a time: the accumulators summed in order
                float d[16];
                uint32_t r[16];
                ptx::tmem_ld_32x32b_x16(tm + ((uint32_t)(quad * 32) << 16) + (uint32_t)m0, r);
                ptx::tmem_ld_wait();
                ptx::tmem_ld_fence_regs<16>(r);
#pragma unroll
                for (int i = 0; i < 16; ++i) d[i] = __uint_as_float(r[i]);
#pragma unroll
                for (int a = 1; a < F::NMMA; ++a) {
                    if (a < G) {
                        ptx::tmem_ld_32x32b_x16(tm + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * MP + m0), r);
                        ptx::tmem_ld_wait();
                        ptx::tmem_ld_fence_regs<16>(r);
#pragma unroll
                        for (int i = 0; i < 16; ++i) d[i] += __uint_as_float(r[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + i;
                    if (m >= M) break;
                    if (splits > 1)
                        part[(size_t)m * kNeu] = d[i];
                    else if (SS1_IN((size_t)m * N + n, (int64_t)M * N, kSiteDecY))
                        Y[(size_t)m * N + n] = __float2bfloat16_rn(FP8 ? sc * d[i] : d[i]);
                }
            }
        } else if (lane == 0 && !*abort_flag) {
            report(status, abort_flag, 4);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tm, F::TMEM_COLS);
    }
    if (splits > 1) {
        // The cluster is this N-block's splits (rank = split). After the first barrier every
        // partial is visible to the cluster; the second keeps each CTA's shared memory alive
        // until its peers have read it.
        ptx::cluster_sync();
        if (warp >= kFirstBuild && warp < kFirstBuild + kEpiWarps) {
            const int t = threadIdx.x - kFirstBuild * 32;   // neuron of the N-block
            const float* part = reinterpret_cast<const float*>(wring) + t;
            const float sc = FP8 && SS1_IN((size_t)nb * kNeu + t, N, kSiteDecScale) ? scale[(size_t)nb * kNeu + t] : 1.0f;
            for (int m = (int)ptx::cluster_ctarank(); m < M && m < MP; m += splits) {
                // every split's partial requested before the first is added: one remote latency
                float pv[16];
#pragma unroll
                for (int s = 0; s < 16; ++s)
                    pv[s] = s < splits ? ptx::ld_cluster_f32(ptx::map_to_rank(part + (size_t)m * kNeu, (uint32_t)s)) : 0.f;
                float v = 0.f;
#pragma unroll
                for (int s = 0; s < 16; ++s)
                    if (s < splits) v += pv[s];   // in split order
                if (SS1_IN((size_t)m * N + (size_t)nb * kNeu + t, (int64_t)M * N, kSiteDecY))
                    Y[(size_t)m * N + (size_t)nb * kNeu + t] = __float2bfloat16_rn(FP8 ? sc * v : v);
            }
        }
        ptx::cluster_sync();
    }
}

// Wc as [N rows x Kc columns]: bf16 with [128 x 64] boxes and the 128-byte swizzle, or E4M3
// codes (one byte each) with [128 x 64] boxes and the 64-byte swizzle.
bool make_map_w(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, bool fp8) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (fp8 ? 1 : 2)};
    cuuint32_t box[2] = {kStageC, kNeu};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// X as [M rows x K] with [16 rows x BK] boxes, no swizzle (chunk mode; rows past M read as zero).
bool make_map_x(CUtensorMap* map, const void* base, uint64_t K, uint64_t M, uint32_t bi) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {K, M};
    cuuint64_t strides[1] = {K * 2};
    cuuint32_t box[2] = {bi, (cuuint32_t)kXChunkRows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MP, int C, bool FP8>
cudaError_t launch_cfg(const ss1_layer& L, const void* X, const void* Wc, const float* scale, void* Y, int64_t M,
                       cudaStream_t st) {
    using F = DecCfg<MP, FP8>;
    const void* fn = reinterpret_cast<const void*>(&dec_kernel<MP, C, FP8>);
    const cudaError_t attr_err = smem_attr_once(fn, F::SMEM);
    if (attr_err != cudaSuccess) return attr_err;
    // CTAs per SM that the launch bounds allow; the K-split aims at that many per SM
    const int per_sm = F::MIN_CTAS;
    const ClusterFit fit = cluster_fit(fn, F::SMEM, F::THREADS);
    CUtensorMap mw, mx;
    if (!make_map_w(&mw, Wc, (uint64_t)(L.K / L.c), (uint64_t)L.N, FP8)) return cudaErrorInvalidValue;
    // Chunk mode: up to 16 rows and K-chunks of whole stages; each chunk's X rows then come by
    // TMA into a two-chunk ring and the sketch gathers read shared memory.
    const int Kc = (int)(L.K / L.c);
    const bool whole_chunks = L.S % kStageC == 0;                          // a unit = one K-chunk
    const bool whole_stages = kStageC % L.S == 0 && Kc % kStageC == 0;     // a unit = one stage
    const int ui = whole_chunks ? L.BK : kStageC * L.c;                    // inputs per unit
    const int bi = ui < 256 ? ui : 256;                                    // inputs per TMA box
    // The one-time copy of a CTA's X columns is cheaper where it fits; the ring is for the rest.
    const int nstg0 = (Kc + kStageC - 1) / kStageC;
    const int splits0 = pick_splits(fit, L.NB, (per_sm * L.num_sms) / L.NB, nstg0);
    const int64_t range_max = ((int64_t)(nstg0 + splits0 - 1) / splits0 * kStageC / L.S + 2) * L.BK;   // inputs
    const bool range_fits = L.BK % 8 == 0 && M * range_max * 2 <= F::X_BYTES;
    const int chunked = (MP == kXChunkRows && !range_fits && L.BK % 8 == 0 && (whole_chunks || whole_stages) &&
                         ui <= 512 && ui % bi == 0) ? 1 : 0;
    if (chunked) {
        if (!make_map_x(&mx, X, (uint64_t)L.K, (uint64_t)M, (uint32_t)bi)) return cudaErrorInvalidValue;
    } else {
        mx = mw;   // unused
    }
    // K-splits: about per_sm CTAs per SM over all N-blocks, each with at least one stage (chunk
    // mode: one K-chunk), and at most one cluster's worth per N-block
    const int nstg = (int)((L.K / L.c + kStageC - 1) / kStageC);
    const int units = chunked ? (whole_chunks ? L.KC : nstg) : nstg;
    const int splits = pick_splits(fit, L.NB, (per_sm * L.num_sms) / L.NB, units);
    // programmatic dependent launch: the CTAs may start while the previous kernel finishes; the
    // splits of one N-block form a cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)L.NB, (unsigned)splits);
    cfg.blockDim = dim3(F::THREADS);
    cfg.dynamicSmemBytes = F::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = (unsigned)splits;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = splits > 1 ? 2 : 1;
    note_launch(FP8 ? "dec_fp8" : "dec", cfg.gridDim.x, cfg.gridDim.y, splits, F::THREADS, F::SMEM, &fit);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, dec_kernel<MP, C, FP8>, mw, mx, (const __nv_bfloat16*)X,
                                             (__nv_bfloat16*)Y, (const uint16_t*)L.d_src, scale, (int)M, (int)L.K,
                                             (int)L.N, L.S, L.KC, splits, chunked, ui, bi, L.status_dev);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int MP, bool FP8>
cudaError_t launch_c(const ss1_layer& L, const void* X, const void* Wc, const float* scale, void* Y, int64_t M,
                     cudaStream_t st) {
    switch (L.c) {
        case 1: return launch_cfg<MP, 1, FP8>(L, X, Wc, scale, Y, M, st);
        case 2: return launch_cfg<MP, 2, FP8>(L, X, Wc, scale, Y, M, st);
        case 4: return launch_cfg<MP, 4, FP8>(L, X, Wc, scale, Y, M, st);
        default: return launch_cfg<MP, 8, FP8>(L, X, Wc, scale, Y, M, st);
    }
}

}  // namespace

bool dec_supported(const ss1_layer& L, int64_t M) {
    if (M < 1 || M > 64) return false;
    if (L.BN != kNeu) return false;
    if (L.K % 8 != 0 || (L.K / L.c) % 8 != 0) return false;
    return true;
}

cudaError_t launch_dec(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    if (M <= 16) return launch_c<16, false>(L, X, Wc, nullptr, Y, M, st);
    if (M <= 32) return launch_c<32, false>(L, X, Wc, nullptr, Y, M, st);
    return launch_c<64, false>(L, X, Wc, nullptr, Y, M, st);
}

bool dec_fp8_supported(const ss1_layer& L, int64_t M) {
    return dec_supported(L, M) && (L.K / L.c) % 16 == 0;   // TMA: rows of Kc bytes, a multiple of 16
}

cudaError_t launch_dec_fp8(const ss1_layer& L, const void* X, const void* Wq, const float* scale, void* Y, int64_t M,
                           cudaStream_t st) {
    if (M <= 16) return launch_c<16, true>(L, X, Wq, scale, Y, M, st);
    if (M <= 32) return launch_c<32, true>(L, X, Wq, scale, Y, M, st);
    return launch_c<64, true>(L, X, Wq, scale, Y, M, st);
}

}  // namespace ss1
