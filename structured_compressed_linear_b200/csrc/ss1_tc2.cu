// Tensor-core SS1 forward for sm_100a, transposed tile: D^T[neurons x rows] = Wc_nb * Xs_nb^T.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": the input is sketched by signed hashed additions and the sketch is multiplied
// with the compressed weights. This kernel keeps the sketch on chip and feeds it to tcgen05.
//
// Tile: 128 neurons (one N-block, UMMA M = 128) x 256 rows of X (UMMA N = 256). One UMMA N of
// 256 is what lets the tensor pipe run near its peak; the operands of one instruction must
// share one hash, and the rows of X do, the neurons of two blocks do not.
// Per K-chunk kc:
//   * TMA warp   : X rows [m0, m0+256) x chunk -> 16 KB smem panels [128 rows x 64 k] (128B
//                  swizzle); Wc[nb*128:+128, kc*S:+S] -> K-major panels; the chunk's gather
//                  table (TMEM column and bf16x2 multiplier per source) -> smem (bulk copy).
//   * MMA thread : tcgen05.cp copies every X panel into TMEM (row r -> lane r % 128, one
//                  32-bit column per pair of inputs), two TMEM buffers per row half when they
//                  fit; then issues S/16 tcgen05.mma (M=128, N=256, K=16) per chunk.
//   * 8 sketch warps (thread = row of the tile): for slot s, Xs[row, s] = sum_j sign_j *
//                  X[row, k_j], gathered with tcgen05.ld from TMEM and accumulated with bf16x2
//                  FMAs whose multiplier keeps the half of the word that holds k_j; the two
//                  halves are folded, rounded once per add, and written as the K-major UMMA B
//                  operand in shared memory. No shared-memory bank is touched for the gather.
//   * epilogue   : tcgen05.ld.16x256b (mma fragment layout) -> bf16 -> stmatrix.trans into a
//                  128B-swizzled [rows x neurons] staging tile -> TMA store of Y.
// Every mbarrier wait is bounded; a wait that runs out sets the CTA's abort flag and the
// handle's status word, drains the copies and MMAs in flight and returns (no trap).
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace ss1 {

// shared with ss1_tc.cu (tensor-map encoding through the driver entry point)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

constexpr int kNeu = 128;        // neurons per tile (UMMA M) = the N-block
constexpr int kRows = 256;       // rows of X per tile (UMMA N)
constexpr int kWarps = 10;       // warp 0 TMA, warp 1 copy+MMA, warps 2..9 sketch (2..5 also epilogue)
constexpr int kThreads = kWarps * 32;
constexpr int kSketchWarps = 8;
constexpr int kXPanel = 128 * 128;   // bytes of one [128 rows x 64 inputs] bf16 panel
constexpr uint32_t kAccCols = 256;   // TMEM columns of the accumulator
constexpr uint64_t kWaitNs = 2000000000ull;

template <int BK, int C>
struct Cfg {
    static constexpr int S = BK / C;
    static constexpr int SP = S < 64 ? S : 64;          // slots per panel (one swizzle row)
    static constexpr int NSP = S / SP;                  // slot panels per chunk
    static constexpr int RB = 2 * SP;                   // bytes per row of a panel
    static constexpr uint32_t LAYOUT = SP == 64 ? ptx::kLayoutSW128 : (SP == 32 ? ptx::kLayoutSW64 : ptx::kLayoutSW32);
    static constexpr int SBO = 8 * RB;
    static constexpr int W_PANEL = kNeu * RB;
    static constexpr int B_PANEL = kRows * RB;
    static constexpr int XPH = BK / 64;                 // X panels per row half per chunk
    static constexpr int NXB = BK <= 128 ? 2 : 1;       // TMEM X buffers
    static constexpr int XCOLS = BK / 2;                // TMEM columns per row half per buffer
    static constexpr int TAB = 2 * BK * 4;              // bytes of one (nb, kc) gather table
    static constexpr int NXS = 4, NWS = 3, NBS = 2, NTS = 2;
    static constexpr int OFF_X = 0;
    static constexpr int OFF_W = OFF_X + NXS * kXPanel;
    static constexpr int OFF_B = OFF_W + NWS * W_PANEL;
    static constexpr int OFF_T = OFF_B + NBS * B_PANEL;
    static constexpr int OFF_A = OFF_T + NTS * TAB;                 // per-warp TMEM address tables
    static constexpr int OFF_BAR = OFF_A + kSketchWarps * BK * 4;
    static constexpr int NBAR = 2 * NXS + 2 * NWS + 2 * NBS + 2 * NTS + 4 * NXB + 1;
    static constexpr int USED = OFF_BAR + NBAR * 8 + 16;
    // at least 120 KB so that one CTA owns the SM (it allocates all 512 TMEM columns)
    static constexpr int SMEM = (USED + 1024 > 120 * 1024) ? USED + 1024 : 120 * 1024;
    static_assert(S % 16 == 0 && S >= 16 && C >= 2, "UMMA K-steps of 16, sketch only for c >= 2");
    static_assert(BK % 64 == 0 && BK <= 256, "X panels of 64 inputs");
    static_assert(kAccCols + 2 * NXB * XCOLS <= 512, "TMEM budget");
    static_assert(kRows * kNeu * 2 <= NXS * kXPanel, "epilogue staging overlays the X ring");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void report(int32_t* status, volatile int* abort_flag, int site) {
    *abort_flag = 1;
    *(volatile int32_t*)status = (kStatusKernelTC << 8) | (0x40 + site);
    __threadfence_system();
}

// Waits for the last `depth` phases of a ring of `n` full-barriers ending at `issued`
// (used only to drain copies in flight after an abort).
__device__ __forceinline__ void drain_ring(uint64_t* full, int n, int issued, int depth) {
    volatile int no_abort = 0;
    for (int i = (issued - depth > 0 ? issued - depth : 0); i < issued; ++i)
        ptx::mbar_wait(&full[i % n], (i / n) & 1, &no_abort, kWaitNs);
}

template <int RB>
__device__ __forceinline__ uint32_t kmajor_off(int row, int col) {
    const uint32_t chunk = (uint32_t)(col >> 3) ^ (uint32_t)(((row * RB) >> 7) & (RB / 16 - 1));
    return (uint32_t)(row * RB) + (chunk << 4) + (uint32_t)(col & 7) * 2u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo_f32, uint32_t hi_f32) {
    __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(lo_f32), __uint_as_float(hi_f32));
    return *reinterpret_cast<uint32_t*>(&b);
}

template <int BK, int C>
__global__ void __launch_bounds__(kThreads, 1)
    tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const __grid_constant__ CUtensorMap tmap_y, const uint32_t* __restrict__ gather, int KC,
               int32_t* status) {
    using F = Cfg<BK, C>;
    constexpr int S = F::S, SP = F::SP, NSP = F::NSP, NXS = F::NXS, NWS = F::NWS, NBS = F::NBS, NTS = F::NTS;
    constexpr int NXB = F::NXB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xring = smem + F::OFF_X;
    uint8_t* wring = smem + F::OFF_W;
    uint8_t* bring = smem + F::OFF_B;
    uint8_t* tring = smem + F::OFF_T;
    uint32_t* atab = reinterpret_cast<uint32_t*>(smem + F::OFF_A);
    uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + F::OFF_BAR);
    uint64_t* x_empty = x_full + NXS;
    uint64_t* w_full = x_empty + NXS;
    uint64_t* w_empty = w_full + NWS;
    uint64_t* b_full = w_empty + NWS;
    uint64_t* b_empty = b_full + NBS;
    uint64_t* t_full = b_empty + NBS;
    uint64_t* t_empty = t_full + NTS;
    uint64_t* tx_full = t_empty + NTS;       // [NXB * 2], index xb * 2 + half
    uint64_t* tx_free = tx_full + 2 * NXB;
    uint64_t* acc_full = tx_free + 2 * NXB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nb = blockIdx.x;
    const int m0 = blockIdx.y * kRows;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NXS; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], 1); }
        for (int i = 0; i < NWS; ++i) { ptx::mbar_init(&w_full[i], 1); ptx::mbar_init(&w_empty[i], 1); }
        for (int i = 0; i < NBS; ++i) { ptx::mbar_init(&b_full[i], 32 * kSketchWarps); ptx::mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < NTS; ++i) { ptx::mbar_init(&t_full[i], 1); ptx::mbar_init(&t_empty[i], 32 * kSketchWarps); }
        for (int i = 0; i < 2 * NXB; ++i) { ptx::mbar_init(&tx_full[i], 1); ptx::mbar_init(&tx_free[i], 128); }
        ptx::mbar_init(acc_full, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_w);
        ptx::prefetch_tmap(&tmap_y);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tm = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int xp = 0, wp = 0, tp = 0;
            for (int kc = 0; kc < KC && !*abort_flag; ++kc) {
                const int ti = kc % NTS;
                if (!ptx::mbar_wait(&t_empty[ti], ((kc / NTS) & 1) ^ 1, abort_flag, kWaitNs)) { report(status, abort_flag, 1); break; }
                ptx::mbar_arrive_expect_tx(&t_full[ti], F::TAB);
                ptx::bulk_load(tring + ti * F::TAB, gather + ((size_t)nb * KC + kc) * 2 * BK, F::TAB, &t_full[ti]);
                ++tp;
                bool ok = true;
                for (int h = 0; h < 2 && ok; ++h)
                    for (int p = 0; p < F::XPH; ++p) {
                        const int slot = xp % NXS;
                        if (!ptx::mbar_wait(&x_empty[slot], ((xp / NXS) & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; break; }
                        ptx::mbar_arrive_expect_tx(&x_full[slot], kXPanel);
                        ptx::tma_load_2d(xring + slot * kXPanel, &tmap_x, &x_full[slot], kc * BK + 64 * p, m0 + 128 * h);
                        ++xp;
                    }
                if (!ok) { report(status, abort_flag, 2); break; }
                for (int sp = 0; sp < NSP; ++sp) {
                    const int wi = wp % NWS;
                    if (!ptx::mbar_wait(&w_empty[wi], ((wp / NWS) & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&w_full[wi], F::W_PANEL);
                    ptx::tma_load_2d(wring + wi * F::W_PANEL, &tmap_w, &w_full[wi], kc * S + sp * SP, nb * kNeu);
                    ++wp;
                }
                if (!ok) { report(status, abort_flag, 3); break; }
            }
            if (*abort_flag) {   // every issued copy must land before the CTA may exit
                drain_ring(x_full, NXS, xp, NXS);
                drain_ring(w_full, NWS, wp, NWS);
                drain_ring(t_full, NTS, tp, NTS);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ TMEM copy + MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kNeu, kRows);
            int xp = 0;
            bool ok = true;
            for (int it = 0; it <= KC && ok; ++it) {
                if (it < KC) {
                    const int xb = it % NXB;
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!ptx::mbar_wait(&tx_free[xb * 2 + h], ((it / NXB) & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; report(status, abort_flag, 4); break; }
                        ptx::tc_fence_after();
                        for (int p = 0; p < F::XPH; ++p) {
                            const int slot = xp % NXS;
                            if (!ptx::mbar_wait(&x_full[slot], (xp / NXS) & 1, abort_flag, kWaitNs)) { ok = false; report(status, abort_flag, 5); break; }
                            const uint32_t col = kAccCols + (uint32_t)((xb * 2 + h) * F::XCOLS + p * 32);
                            const uint32_t src = ptx::smem_u32(xring + slot * kXPanel);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                ptx::tmem_cp_128x256b(tm + col + q * 8, ptx::smem_desc(src + q * 32, 16, 1024, ptx::kLayoutSW128));
                            ptx::umma_commit(&x_empty[slot]);
                            ++xp;
                        }
                        if (ok) ptx::umma_commit(&tx_full[xb * 2 + h]);
                    }
                }
                if (it >= 1 && ok) {
                    const int kc = it - 1;
                    for (int sp = 0; sp < NSP; ++sp) {
                        const int wc = kc * NSP + sp;
                        const int wi = wc % NWS, bi = wc % NBS;
                        if (!ptx::mbar_wait(&w_full[wi], (wc / NWS) & 1, abort_flag, kWaitNs) ||
                            !ptx::mbar_wait(&b_full[bi], (wc / NBS) & 1, abort_flag, kWaitNs)) {
                            ok = false;
                            report(status, abort_flag, 6);
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t a0 = ptx::smem_u32(wring + wi * F::W_PANEL);
                        const uint32_t b0 = ptx::smem_u32(bring + bi * F::B_PANEL);
#pragma unroll
                        for (int kk = 0; kk < SP / 16; ++kk)
                            ptx::umma_bf16_ss(tm, ptx::smem_desc(a0 + kk * 32, 16, F::SBO, F::LAYOUT),
                                              ptx::smem_desc(b0 + kk * 32, 16, F::SBO, F::LAYOUT), idesc,
                                              (wc > 0 || kk > 0) ? 1u : 0u);
                        ptx::umma_commit(&w_empty[wi]);
                        ptx::umma_commit(&b_empty[bi]);
                    }
                }
            }
            ptx::umma_commit(acc_full);
            if (*abort_flag) {
                volatile int no_abort = 0;
                ptx::mbar_wait(acc_full, 0, &no_abort, kWaitNs);   // copies and MMAs in flight finish
            }
        }
    } else {
        // ------------------------------------------------------------------ sketch warps
        const int sw = warp - 2;                     // 0..7
        const int half = sw >> 2;                    // rows [128*half, 128*half + 128) of the tile
        const int quad = warp & 3;                   // TMEM lanes 32*quad .. +31
        const int row = half * 128 + quad * 32 + lane;
        uint32_t* mytab = atab + sw * BK;
        for (int kc = 0; kc < KC; ++kc) {
            const int xb = kc % NXB, ti = kc % NTS;
            if (!ptx::mbar_wait(&tx_full[xb * 2 + half], (kc / NXB) & 1, abort_flag, kWaitNs) ||
                !ptx::mbar_wait(&t_full[ti], (kc / NTS) & 1, abort_flag, kWaitNs)) {
                report(status, abort_flag, 7);
                break;
            }
            ptx::tc_fence_after();
            const uint32_t xbase = tm + ((uint32_t)(quad * 32) << 16) + kAccCols + (uint32_t)((xb * 2 + half) * F::XCOLS);
            const uint32_t* tcol = reinterpret_cast<const uint32_t*>(tring + ti * F::TAB);
            const uint32_t* tmul = tcol + BK;
            __syncwarp();
            for (int i = lane; i < BK; i += 32) mytab[i] = xbase + tcol[i];
            __syncwarp();
            bool ok = true;
            for (int sp = 0; sp < NSP; ++sp) {
                const int wc = kc * NSP + sp;
                const int bi = wc % NBS;
                if (!ptx::mbar_wait(&b_empty[bi], ((wc / NBS) & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; break; }
                uint8_t* bp = bring + bi * F::B_PANEL;
#pragma unroll 1
                for (int s8 = 0; s8 < SP / 8; ++s8) {
                    const int e0 = (sp * SP + s8 * 8) * C;   // first source of these 8 slots
                    uint32_t w[8 * C];
#pragma unroll
                    for (int q = 0; q < 2 * C; ++q) {
                        const uint4 t4 = *reinterpret_cast<const uint4*>(mytab + e0 + 4 * q);
                        w[4 * q + 0] = ptx::tmem_ld_32x32b_x1(t4.x);
                        w[4 * q + 1] = ptx::tmem_ld_32x32b_x1(t4.y);
                        w[4 * q + 2] = ptx::tmem_ld_32x32b_x1(t4.z);
                        w[4 * q + 3] = ptx::tmem_ld_32x32b_x1(t4.w);
                    }
                    ptx::tmem_ld_wait();
                    __nv_bfloat162 acc[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
                    for (int q = 0; q < 2 * C; ++q) {
                        const uint4 m4 = *reinterpret_cast<const uint4*>(tmul + e0 + 4 * q);
                        const uint32_t mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int idx = 4 * q + j;
                            acc[idx / C] = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&w[idx]),
                                                   *reinterpret_cast<const __nv_bfloat162*>(&mm[j]), acc[idx / C]);
                        }
                    }
                    uint32_t out[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint32_t a = *reinterpret_cast<uint32_t*>(&acc[2 * p]);
                        const uint32_t b = *reinterpret_cast<uint32_t*>(&acc[2 * p + 1]);
                        const uint32_t lo = __byte_perm(a, b, 0x5410), hi = __byte_perm(a, b, 0x7632);
                        __nv_bfloat162 r = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&lo),
                                                   *reinterpret_cast<const __nv_bfloat162*>(&hi));
                        out[p] = *reinterpret_cast<uint32_t*>(&r);
                    }
                    *reinterpret_cast<uint4*>(bp + kmajor_off<F::RB>(row, s8 * 8)) = make_uint4(out[0], out[1], out[2], out[3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(&b_full[bi]);
            }
            if (!ok) { report(status, abort_flag, 8); break; }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&tx_free[xb * 2 + half]);
            ptx::mbar_arrive(&t_empty[ti]);
        }

        // ------------------------------------------------------------------ epilogue (warps 2..5)
        if (warp <= 5) {
            bool ok = ptx::mbar_wait(acc_full, 0, abort_flag, kWaitNs);
            if (!ok) report(status, abort_flag, 9);
            ptx::tc_fence_after();
            ok = __all_sync(0xffffffffu, ok && !*abort_flag);
            uint8_t* stage = xring;   // [2 boxes][256 rows][64 neurons] bf16, 128B-swizzled
            if (ok) {
                const int mi = lane >> 3, mj = lane & 7;
                const int n = quad * 32 + mi * 8;          // first neuron of this thread's 8x8 matrix
                const int box = n >> 6, nin = n & 63;
#pragma unroll 1
                for (int c0 = 0; c0 < kRows; c0 += 8) {
                    uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
                    ptx::tmem_ld_16x256b(tm + ((uint32_t)(quad * 32) << 16) + c0, r0, r1, r2, r3);
                    ptx::tmem_ld_16x256b(tm + ((uint32_t)(quad * 32 + 16) << 16) + c0, r4, r5, r6, r7);
                    ptx::tmem_ld_wait();
                    const int rrow = c0 + mj;
                    const uint32_t off = (uint32_t)(box * (kRows * 128) + rrow * 128) +
                                         ((uint32_t)((nin >> 3) ^ (rrow & 7)) << 4);
                    ptx::stmatrix_x4_trans(ptx::smem_u32(stage + off), pack_bf16x2(r0, r1), pack_bf16x2(r2, r3),
                                           pack_bf16x2(r4, r5), pack_bf16x2(r6, r7));
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::named_barrier_sync(1, 128);
            if (warp == 2 && lane == 0 && !*abort_flag) {
                ptx::tma_store_2d(&tmap_y, stage, nb * kNeu, m0);
                ptx::tma_store_2d(&tmap_y, stage + kRows * 128, nb * kNeu + 64, m0);
                ptx::tma_store_commit();
                ptx::tma_store_wait0();
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tm, 512);
    }
}

bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle sw) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BK, int C>
cudaError_t launch_cfg(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    using F = Cfg<BK, C>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(tc2_kernel<BK, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const CUtensorMapSwizzle wsw = F::SP == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                               : (F::SP == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    CUtensorMap mx, mw, my;
    if (!make_map(&mx, X, (uint64_t)L.K, (uint64_t)M, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mw, Wc, (uint64_t)(L.K / L.c), (uint64_t)L.N, F::SP, kNeu, wsw) ||
        !make_map(&my, Y, (uint64_t)L.N, (uint64_t)M, 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    dim3 grid((unsigned)L.NB, (unsigned)((M + kRows - 1) / kRows));
    tc2_kernel<BK, C><<<grid, kThreads, F::SMEM, st>>>(mx, mw, my, L.d_gather, L.KC, L.status_dev);
    return cudaGetLastError();
}

}  // namespace

bool tc2_supported(const ss1_layer& L) {
    if (L.BN != kNeu || L.c < 2) return false;
    if (!(L.BK == 64 || L.BK == 128 || L.BK == 256)) return false;
    if (L.S < 16 || L.S % 16 != 0) return false;
    if (L.K % 8 != 0 || (L.K / L.c) % 8 != 0 || L.N % 8 != 0) return false;
    return true;
}

cudaError_t launch_tc2(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    if ((M + kRows - 1) / kRows > 65535) return cudaErrorInvalidValue;
#define SS1_TC2_CASE(bk, cc) \
    if (L.BK == bk && L.c == cc) return launch_cfg<bk, cc>(L, X, Wc, Y, M, st);
    SS1_TC2_CASE(64, 2)
    SS1_TC2_CASE(64, 4)
    SS1_TC2_CASE(128, 2)
    SS1_TC2_CASE(128, 4)
    SS1_TC2_CASE(128, 8)
    SS1_TC2_CASE(256, 2)
    SS1_TC2_CASE(256, 4)
    SS1_TC2_CASE(256, 8)
#undef SS1_TC2_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ss1
