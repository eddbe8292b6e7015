// Tensor-core SS1 forward for sm_100a at c = 1: TMA -> tcgen05.mma (TMEM accumulator) -> Y.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": the input is sketched (signed hashed additions shrink it by the compression
// factor c) and then multiplied with the compressed weights. At c = 1 the hash is the identity
// with all signs +1, so the layer is the dense product Y = X Wc^T and the X tile itself is the
// A operand. (c >= 2 runs in ss1_tc3.cu, or in ss1_tc2.cu for the shapes tc3 does not take;
// launch_tc below chooses.)
//
// Two kernels. Where N is a multiple of 256 and the layer spans more than one wave of 128 x 128
// tiles, tcw_kernel (below): persistent CTAs, 128 x 256 output tiles, two TMEM accumulators.
// Otherwise tc_kernel: one CTA computes a 128-row x 128-column
// output tile = rows [m0, m0+128) of N-block nb (BN = 128 = the UMMA N). Per K-chunk kc (BK inputs):
//   * TMA warp      : X[m0:+128, kc*BK:+BK] -> smem (128B-swizzled, 64-column panels) and
//                     Wc[nb*128:+128, kc*BK:+BK] -> smem (K-major, 128B swizzle).
//   * MMA thread    : BK/16 x tcgen05.mma.kind::f16 (M=128, N=128, K=16) into one TMEM
//                     accumulator; tcgen05.commit releases the stage.
//   * epilogue warps: read the fp32 accumulator with tcgen05.ld, round to bf16 and store Y.
// Every mbarrier wait is bounded; a wait that runs out sets the CTA's abort flag and the
// handle's status word, drains the copies and MMAs in flight and returns (no trap).
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

namespace ss1 {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

constexpr int kBM = 128;         // rows per tile (UMMA M)
constexpr int kBN = 128;         // N-block size handled (UMMA N)
constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kSmemBudget = 200 * 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
[[maybe_unused]] constexpr int kSiteTcY = kSiteHashSlot + 1;   // checked build: the Y stores of both kernels here

template <int BK>
struct Cfg {
    static constexpr int S = BK;                        // c = 1: one compressed column per input
    static constexpr int X_BYTES = kBM * BK * 2;
    static constexpr int W_BYTES = kBN * S * 2;
    static constexpr int RB = S >= 64 ? 128 : 2 * S;   // bytes per row inside one swizzle panel
    static constexpr int PANEL = 128 * RB;              // bytes of one 128-row panel
    static constexpr uint32_t LAYOUT = S >= 64 ? ptx::kLayoutSW128 : (S == 32 ? ptx::kLayoutSW64 : ptx::kLayoutSW32);
    static constexpr int SBO = 8 * RB;                  // byte distance of consecutive 8-row groups

    static constexpr int stage_pick(bool want_x) {
        int best_x = 1, best_w = 1, best_score = -1;
        for (int nx = 1; nx <= 4; ++nx)
            for (int nw = 1; nw <= 4; ++nw) {
                const int bytes = nx * X_BYTES + nw * W_BYTES;
                if (bytes > kSmemBudget) continue;
                const int score = (nx < nw ? nx : nw) * 16 + nx + nw;
                if (score > best_score) { best_score = score; best_x = nx; best_w = nw; }
            }
        return want_x ? best_x : best_w;
    }
    static constexpr int NX = stage_pick(true);
    static constexpr int NW = stage_pick(false);
    static constexpr int NBAR = 2 * NX + 2 * NW + 1;
    static constexpr int SMEM = NX * X_BYTES + NW * W_BYTES + NBAR * 8 + 16 + 1024;
    static_assert(S % 16 == 0 && S >= 16, "UMMA K-steps of 16");
    static_assert(BK % 64 == 0, "X panels of 64 columns");
};

__device__ __forceinline__ void report(int32_t* status, volatile int* abort_flag, int site) {
    *abort_flag = 1;
    *(volatile int32_t*)status = (kStatusKernelTC << 8) | site;
    __threadfence_system();
}

template <int BK>
__global__ void __launch_bounds__(kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
              __nv_bfloat16* __restrict__ Y, int M, int N, int KC, int32_t* status) {
    using F = Cfg<BK>;
    constexpr int S = F::S, NX = F::NX, NW = F::NW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xs = smem;
    uint8_t* ws = xs + NX * F::X_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(ws + NW * F::W_BYTES);
    uint64_t* x_full = bars;
    uint64_t* x_empty = x_full + NX;
    uint64_t* w_full = x_empty + NX;
    uint64_t* aw_empty = w_full + NW;
    uint64_t* acc_full = aw_empty + NW;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nb = blockIdx.x;
    const int m0 = blockIdx.y * kBM;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NX; ++i) {
            ptx::mbar_init(&x_full[i], 1);
            ptx::mbar_init(&x_empty[i], 1);
        }
        for (int i = 0; i < NW; ++i) {
            ptx::mbar_init(&w_full[i], 1);
            ptx::mbar_init(&aw_empty[i], 1);
        }
        ptx::mbar_init(acc_full, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, kBN);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_w);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_acc = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last_x = -1, last_w = -1;
            for (int kc = 0; kc < KC; ++kc) {
                const int xi = kc % NX, wi = kc % NW;
                if (!ptx::mbar_wait(&x_empty[xi], ((kc / NX) & 1) ^ 1, abort_flag, kWaitLimitNs)) {
                    report(status, abort_flag, 1);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&x_full[xi], F::X_BYTES);
#pragma unroll
                for (int p = 0; p < BK / 64; ++p)
                    ptx::tma_load_2d(xs + xi * F::X_BYTES + p * 128 * 128, &tmap_x, &x_full[xi], kc * BK + p * 64, m0);
                last_x = kc;
                if (!ptx::mbar_wait(&aw_empty[wi], ((kc / NW) & 1) ^ 1, abort_flag, kWaitLimitNs)) {
                    report(status, abort_flag, 2);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&w_full[wi], F::W_BYTES);
#pragma unroll
                for (int p = 0; p < (S + 63) / 64; ++p)
                    ptx::tma_load_2d(ws + wi * F::W_BYTES + p * F::PANEL, &tmap_w, &w_full[wi], kc * S + p * 64,
                                     nb * kBN);
                last_w = kc;
            }
            if (*abort_flag) {
                // drain: every issued copy must land before the CTA may exit
                volatile int no_abort = 0;
                for (int kc = (last_x - NX + 1 > 0 ? last_x - NX + 1 : 0); kc <= last_x; ++kc)
                    ptx::mbar_wait(&x_full[kc % NX], (kc / NX) & 1, &no_abort, kWaitLimitNs);
                for (int kc = (last_w - NW + 1 > 0 ? last_w - NW + 1 : 0); kc <= last_w; ++kc)
                    ptx::mbar_wait(&w_full[kc % NW], (kc / NW) & 1, &no_abort, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, kBN);
            for (int kc = 0; kc < KC; ++kc) {
                const int wi = kc % NW;
                const uint32_t ph = (kc / NW) & 1;
                if (!ptx::mbar_wait(&w_full[wi], ph, abort_flag, kWaitLimitNs)) { report(status, abort_flag, 3); break; }
                if (!ptx::mbar_wait(&x_full[kc % NX], (kc / NX) & 1, abort_flag, kWaitLimitNs)) {
                    report(status, abort_flag, 4);
                    break;
                }
                const uint8_t* a_tile = xs + (kc % NX) * F::X_BYTES;
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_u32(a_tile);
                const uint32_t b_base = ptx::smem_u32(ws + wi * F::W_BYTES);
#pragma unroll
                for (int kk = 0; kk < S / 16; ++kk) {
                    constexpr int per_panel = F::RB / 2;
                    const uint32_t off = (uint32_t)((kk * 16) / per_panel) * F::PANEL + (uint32_t)((kk * 16) % per_panel) * 2u;
                    const uint64_t ad = ptx::smem_desc(a_base + off, 16, F::SBO, F::LAYOUT);
                    const uint64_t bd = ptx::smem_desc(b_base + off, 16, F::SBO, F::LAYOUT);
                    ptx::umma_bf16_ss(tmem_acc, ad, bd, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::umma_commit(&aw_empty[wi]);
                ptx::umma_commit(&x_empty[kc % NX]);
            }
            ptx::umma_commit(acc_full);
            if (*abort_flag) {
                volatile int no_abort = 0;
                ptx::mbar_wait(acc_full, 0, &no_abort, kWaitLimitNs);  // MMAs in flight finish before exit
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;              // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;       // row of the tile owned by this thread
        bool ok = ptx::mbar_wait(acc_full, 0, abort_flag, kWaitLimitNs);
        if (!ok) report(status, abort_flag, 7);
        ptx::tc_fence_after();
        ok = __all_sync(0xffffffffu, ok && !*abort_flag);   // tcgen05.ld is warp-collective
        if (ok) {
            const int m = m0 + row;
            __nv_bfloat16* yrow = Y + (size_t)m * N + (size_t)nb * kBN;
#pragma unroll 1
            for (int col0 = 0; col0 < kBN; col0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld_32x32b_x32(tmem_acc + ((uint32_t)(quad * 32) << 16) + (uint32_t)col0, r);
                ptx::tmem_ld_wait();
                if (m < M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 o;
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[q * 8 + 2 * t]),
                                                                     __uint_as_float(r[q * 8 + 2 * t + 1]));
                            ow[t] = *reinterpret_cast<uint32_t*>(&b);
                        }
                        if (SS1_SPAN_IN(yrow + col0 + q * 8 - Y, 8, (int64_t)M * N, kSiteTcY))
                            *reinterpret_cast<uint4*>(yrow + col0 + q * 8) = o;
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_acc, kBN);
    }
}

// ---------------------------------------------------------------------------- wide persistent kernel
// c = 1 with N a multiple of 256: one CTA per SM walks the output tiles of 128 rows x 256 columns
// (tile t = blockIdx.x + i * gridDim.x, its 256 columns fastest, so the CTAs running at once
// share X row panels in L2). UMMA N = 256 halves the shared-memory bytes the tensor pipe reads
// per flop against N = 128 (A is read once for twice the columns), which is what holds the
// 128 x 128 tile below the tensor rate. The K loop runs in stages of 64 columns (X 16 KB + W
// 32 KB) through a 4-deep ring, across tile boundaries; two TMEM accumulators of 256 columns let
// the epilogue warps store one tile while the MMA thread fills the other.
constexpr int kWN = 256;                         // output columns per tile (UMMA N)
constexpr int kWK = 64;                          // K columns per stage
constexpr int kWRing = 4;                        // stages in the ring
constexpr int kWXBytes = kBM * kWK * 2;          // 16 KB
constexpr int kWWBytes = kWN * kWK * 2;          // 32 KB
constexpr int kWStage = kWXBytes + kWWBytes;     // 48 KB, a multiple of the 1 KB swizzle atom
constexpr int kWNBar = 2 * kWRing + 2 + 2 + 1;
constexpr int kWSmem = kWRing * kWStage + kWNBar * 8 + 16 + 1024;
static_assert(kWSmem <= 227 * 1024, "shared memory of one CTA");

__global__ void __launch_bounds__(kThreads, 1)
    tcw_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               __nv_bfloat16* __restrict__ Y, int M, int N, int K, int num_tiles, int tiles_n, int32_t* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWRing * kWStage);
    uint64_t* full = bars;                   // [kWRing] a stage's X and W tiles have landed
    uint64_t* empty = full + kWRing;         // [kWRing] the stage's UMMAs have completed
    uint64_t* acc_full = empty + kWRing;     // [2] an accumulator holds a finished tile
    uint64_t* acc_empty = acc_full + 2;      // [2] the epilogue has read an accumulator
    uint64_t* mma_done = acc_empty + 2;      // time-out path: the UMMAs in flight have completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int KS = (K + kWK - 1) / kWK;      // stages per tile (TMA reads zeros past K)

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWRing; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&acc_full[i], 1);
            ptx::mbar_init(&acc_empty[i], 4);   // one arrival per epilogue warp
        }
        ptx::mbar_init(mma_done, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 2 * kWN);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_w);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                const int m0 = (tile / tiles_n) * kBM, n0 = (tile % tiles_n) * kWN;
                for (int ks = 0; ks < KS; ++ks, ++it) {
                    const int sl = it % kWRing;
                    if (it >= kWRing &&
                        !ptx::mbar_wait(&empty[sl], (uint32_t)(((it / kWRing) - 1) & 1), abort_flag, kWaitLimitNs)) {
                        report(status, abort_flag, 11);
                        break;
                    }
                    uint8_t* st = smem + sl * kWStage;
                    ptx::mbar_arrive_expect_tx(&full[sl], kWStage);
                    ptx::tma_load_2d(st, &tmap_x, &full[sl], ks * kWK, m0);
                    ptx::tma_load_2d(st + kWXBytes, &tmap_w, &full[sl], ks * kWK, n0);
                }
            }
            if (*abort_flag) {   // every issued copy lands before the CTA may exit
                volatile int no_abort = 0;
                for (int j = it > kWRing ? it - kWRing : 0; j < it; ++j)
                    ptx::mbar_wait(&full[j % kWRing], (uint32_t)((j / kWRing) & 1), &no_abort, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, kWN);
            int it = 0, tl = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
                const int a = tl & 1;
                if (tl >= 2 && !ptx::mbar_wait(&acc_empty[a], (uint32_t)(((tl / 2) - 1) & 1), abort_flag, kWaitLimitNs)) {
                    report(status, abort_flag, 12);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(a * kWN);
                for (int ks = 0; ks < KS; ++ks, ++it) {
                    const int sl = it % kWRing;
                    if (!ptx::mbar_wait(&full[sl], (uint32_t)((it / kWRing) & 1), abort_flag, kWaitLimitNs)) {
                        report(status, abort_flag, 13);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t xb = ptx::smem_u32(smem + sl * kWStage);
                    const uint32_t wb = xb + (uint32_t)kWXBytes;
#pragma unroll
                    for (int kk = 0; kk < kWK / 16; ++kk) {   // 16 columns = 32 bytes along the swizzled row
                        const uint64_t ad = ptx::smem_desc(xb + (uint32_t)(kk * 32), 16, 1024, ptx::kLayoutSW128);
                        const uint64_t bd = ptx::smem_desc(wb + (uint32_t)(kk * 32), 16, 1024, ptx::kLayoutSW128);
                        ptx::umma_bf16_ss(acc, ad, bd, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::umma_commit(&empty[sl]);
                }
                if (!ok) break;
                ptx::umma_commit(&acc_full[a]);
            }
            if (*abort_flag) {   // the UMMAs in flight complete before TMEM is released
                ptx::umma_commit(mma_done);
                volatile int no_abort = 0;
                ptx::mbar_wait(mma_done, 0, &no_abort, kWaitLimitNs);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;              // TMEM lanes 32 quad .. 32 quad + 31
        const int row = quad * 32 + lane;
        int tl = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
            const int a = tl & 1;
            bool ok = ptx::mbar_wait(&acc_full[a], (uint32_t)((tl / 2) & 1), abort_flag, kWaitLimitNs);
            if (!ok && lane == 0 && !*abort_flag) report(status, abort_flag, 14);
            ptx::tc_fence_after();
            ok = __all_sync(0xffffffffu, ok && !*abort_flag);   // tcgen05.ld is warp-collective
            if (!ok) break;
            const int m = (tile / tiles_n) * kBM + row;
            __nv_bfloat16* yrow = Y + (size_t)m * N + (size_t)(tile % tiles_n) * kWN;
#pragma unroll 1
            for (int col0 = 0; col0 < kWN; col0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * kWN + col0), r);
                ptx::tmem_ld_wait();
                if (m < M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 o;
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[q * 8 + 2 * t]),
                                                                     __uint_as_float(r[q * 8 + 2 * t + 1]));
                            ow[t] = *reinterpret_cast<uint32_t*>(&b);
                        }
                        if (SS1_SPAN_IN(yrow + col0 + q * 8 - Y, 8, (int64_t)M * N, kSiteTcY))
                            *reinterpret_cast<uint4*>(yrow + col0 + q * 8) = o;
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[a]);   // this warp's lanes of the accumulator are read
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 2 * kWN);
    }
}

// ---------------------------------------------------------------------------- host side

bool make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                 uint32_t box_outer, CUtensorMapSwizzle sw) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BK>
cudaError_t launch_cfg(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    using F = Cfg<BK>;
    constexpr int S = F::S;
    const cudaError_t attr_err = smem_attr_once(reinterpret_cast<const void*>(&tc_kernel<BK>), F::SMEM);
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mx, mw;
    const CUtensorMapSwizzle wsw = S >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (S == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (!make_map_2d(&mx, X, (uint64_t)L.K, (uint64_t)M, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
    if (!make_map_2d(&mw, Wc, (uint64_t)(L.K / L.c), (uint64_t)L.N, S >= 64 ? 64 : S, kBN, wsw))
        return cudaErrorInvalidValue;
    dim3 grid((unsigned)L.NB, (unsigned)((M + kBM - 1) / kBM));
    note_launch("tc", grid.x, grid.y, 1, kThreads, F::SMEM, nullptr);
    tc_kernel<BK><<<grid, kThreads, F::SMEM, st>>>(mx, mw, (__nv_bfloat16*)Y, (int)M, (int)L.N, L.KC, L.status_dev);
    return cudaGetLastError();
}

cudaError_t launch_wide(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    const cudaError_t attr_err = smem_attr_once(reinterpret_cast<const void*>(&tcw_kernel), kWSmem);
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mx, mw;
    if (!make_map_2d(&mx, X, (uint64_t)L.K, (uint64_t)M, kWK, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mw, Wc, (uint64_t)L.K, (uint64_t)L.N, kWK, kWN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int64_t tiles_n = L.N / kWN, tiles = tiles_n * ((M + kBM - 1) / kBM);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, L.num_sms > 0 ? L.num_sms : 148);
    note_launch("tc", grid, 1, 1, kThreads, kWSmem, nullptr);
    tcw_kernel<<<grid, kThreads, kWSmem, st>>>(mx, mw, (__nv_bfloat16*)Y, (int)M, (int)L.N, (int)L.K, (int)tiles,
                                               (int)tiles_n, L.status_dev);
    return cudaGetLastError();
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool tc_supported(const ss1_layer& L) {
    if (L.BN != kBN) return false;
    if (!(L.BK == 64 || L.BK == 128 || L.BK == 256)) return false;
    if (L.S < 16 || L.S % 16 != 0) return false;
    if (L.K % 8 != 0 || (L.K / L.c) % 8 != 0) return false;
    return true;
}

cudaError_t launch_tc(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    if (tc3_supported(L)) return launch_tc3(L, X, Wc, Y, M, nullptr, 0, st);
    if (tc2_supported(L)) return launch_tc2(L, X, Wc, Y, M, st);
    // c >= 2 shapes that tc_supported accepts are all taken above (tc2_supported covers them)
    if (L.c != 1) return cudaErrorInvalidValue;
    // The wide kernel where the 128 x 128 grid would need more than one wave. Below that, twice
    // the CTAs of 128 x 128 tiles stream Wc faster (each SM's TMA rate bounds a CTA there): at
    // M = 64 on 4096 x 4096, 16 wide CTAs took 36 us against 28 us for 32 narrow ones.
    const int64_t wide_tiles = (M + kBM - 1) / kBM * (L.N / kWN);
    if (L.N % kWN == 0 && 2 * wide_tiles > (int64_t)L.num_sms) return launch_wide(L, X, Wc, Y, M, st);
    if ((M + kBM - 1) / kBM > 65535) return cudaErrorInvalidValue;
    if (L.BK == 64) return launch_cfg<64>(L, X, Wc, Y, M, st);
    if (L.BK == 128) return launch_cfg<128>(L, X, Wc, Y, M, st);
    if (L.BK == 256) return launch_cfg<256>(L, X, Wc, Y, M, st);
    return cudaErrorInvalidValue;
}

}  // namespace ss1
