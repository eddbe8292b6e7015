// Tensor-core SS1 forward for sm_100a, transposed tile: D^T[neurons x rows] = Wc_nb * Xs_nb^T.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": the input is sketched by signed hashed additions and the sketch is multiplied
// with the compressed weights. This kernel keeps the sketch on chip and feeds it to tcgen05.
//
// Tile: 128 neurons (one N-block, UMMA M = 128) x 256 rows of X (UMMA N = 256). An UMMA N of
// 256 is what lets the tensor pipe run near its peak, and the operands of one instruction must
// share one hash: rows of X do, neurons of two blocks do not. Persistent CTAs (one per SM)
// walk the tiles with the N-block index fastest, so CTAs running side by side share X in L2.
// Per K-chunk kc of a tile:
//   * X warp     : X rows [m0, m0+256) x 64 inputs per TMA box (32 KB, 128B swizzle) into a
//                  3-slot ring.
//   * Wc warp    : Wc[nb*128:+128, kc*S:+S] with 16-byte cp.async into K-major swizzled panels
//                  (the UMMA A operand), 3-slot ring.
//   * 16 sketch warps. A thread owns rows r and r+128 of the tile (r = TMEM lane). They first
//                  stage the X chunk into TMEM as row pairs: conflict-free 16-byte shared loads,
//                  byte permutes to (X[r][k], X[r+128][k]), tcgen05.st -> column k. Then, for
//                  their quarter of the slots, Xs[., s] = sum_j sign_j * X[., k_j] with one
//                  tcgen05.ld (two rows at once) and one bf16x2 FMA per source, whose TMEM
//                  column and +-1 multiplier come ready-made from the table (L1-resident), and
//                  write both rows as the K-major UMMA B operand (2-slot ring).
//   * MMA warp   : S/16 x tcgen05.mma (M=128, N=256, K=16) per chunk into one accumulator.
//   * 4 epilogue warps: tcgen05.ld.16x256b (mma fragment layout) -> bf16 -> stmatrix.trans into
//                  a private swizzled [32 rows x 32 neurons] staging tile -> 16-byte stores of
//                  Y rows; they release the accumulator as soon as its last column is read.
// Every mbarrier wait is bounded; a wait that runs out sets the CTA's abort flag and the
// handle's status word, drains the copies and MMAs in flight and returns (no trap).
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace ss1 {

// defined in ss1_tc.cu (tensor-map encoding through the driver entry point)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

constexpr int kNeu = 128;        // neurons per tile (UMMA M) = the N-block
constexpr int kRows = 256;       // rows of X per tile (UMMA N)
constexpr int kSketchWarps = 16;
constexpr int kEpiWarps = 4;
constexpr int kFirstSketch = 3;                         // warp 0 X loads, warp 1 Wc loads, warp 2 MMA
constexpr int kFirstEpi = kFirstSketch + kSketchWarps;  // warps 19..22
constexpr int kWarps = kFirstEpi + kEpiWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kXSlot = kRows * 128;    // bytes of one [256 rows x 64 inputs] bf16 TMA box
constexpr int kEpiStage = 32 * 32 * 2; // per epilogue warp: [32 rows x 32 neurons] bf16
constexpr uint32_t kAccCols = 256;     // TMEM columns of the accumulator
constexpr int kBatch = 16;             // sources per gather batch (TMEM loads in flight per wait)
constexpr uint64_t kWaitNs = 2000000000ull;

template <int BK, int C>
struct Cfg {
    static constexpr int S = BK / C;
    static constexpr int SP = S < 64 ? S : 64;          // slots per panel (one swizzle row)
    static constexpr int NSP = S / SP;                  // slot panels per chunk
    static constexpr int SB = kBatch / C;               // slots per gather batch
    static constexpr int NBATCH = SP / SB;              // batches per panel (split over 4 warps)
    static constexpr int RB = 2 * SP;                   // bytes per row of a panel
    static constexpr uint32_t LAYOUT = SP == 64 ? ptx::kLayoutSW128 : (SP == 32 ? ptx::kLayoutSW64 : ptx::kLayoutSW32);
    static constexpr int SBO = 8 * RB;
    static constexpr int W_PANEL = kNeu * RB;
    static constexpr int B_PANEL = kRows * RB;
    static constexpr int XPH = BK / 64;                 // X boxes (64 inputs x 256 rows) per chunk
    static constexpr int NXB = BK <= 128 ? 2 : 1;       // TMEM X buffers (BK row-pair columns each)
    static constexpr int NXS = 3, NBS = 2, NWS = 3;
    static constexpr int TEAMS = NXB;                   // sketch teams: one per TMEM staging buffer
    static constexpr int OFF_X = 0;
    static constexpr int OFF_W = OFF_X + NXS * kXSlot;
    static constexpr int OFF_B = OFF_W + NWS * W_PANEL;
    static constexpr int OFF_E = OFF_B + NBS * B_PANEL;                 // epilogue staging
    static constexpr int OFF_BAR = OFF_E + kEpiWarps * kEpiStage;
    static constexpr int NBAR = 2 * NXS + 2 * NWS + 2 * NBS + 3;
    static constexpr int USED = OFF_BAR + NBAR * 8 + 16;
    // at least 120 KB so that one CTA owns the SM (it allocates all 512 TMEM columns)
    static constexpr int SMEM = (USED + 1024 > 120 * 1024) ? USED + 1024 : 120 * 1024;
    static_assert(S % 16 == 0 && S >= 16 && C >= 2, "UMMA K-steps of 16, sketch only for c >= 2");
    static_assert(BK % 64 == 0 && BK <= 256, "X boxes of 64 inputs");
    static constexpr int GROUPS = 4 / TEAMS;            // slot parts per team (warps per lane quarter)
    static_assert(SB >= 2 && SP % SB == 0 && NBATCH % GROUPS == 0, "gather batches split over a team's slot parts");
    static_assert((NBATCH / GROUPS) % (NBATCH / GROUPS < 2 ? NBATCH / GROUPS : 2) == 0, "load rounds cover a warp's batches");
    static_assert(kAccCols + NXB * BK <= 512, "TMEM budget");
    static_assert(W_PANEL % (32 * 16) == 0, "Wc panel copied in 16-byte pieces by one warp");
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

// Lane 0 waits, the warp follows: one poller per warp instead of 32.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, abort_flag, kWaitNs);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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
    tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __nv_bfloat16* __restrict__ Wc,
               __nv_bfloat16* __restrict__ Y, const uint2* __restrict__ gather_tab, int M, int N, int Kc, int KC,
               int NB, int num_tiles, int32_t* status) {
    using F = Cfg<BK, C>;
    constexpr int S = F::S, SP = F::SP, SB = F::SB, NSP = F::NSP, NXS = F::NXS, NWS = F::NWS, NBS = F::NBS;
    constexpr int NXB = F::NXB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xring = smem + F::OFF_X;
    uint8_t* wring = smem + F::OFF_W;
    uint8_t* bring = smem + F::OFF_B;
    uint8_t* estage = smem + F::OFF_E;
    uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + F::OFF_BAR);
    uint64_t* x_empty = x_full + NXS;
    uint64_t* w_full = x_empty + NXS;
    uint64_t* w_empty = w_full + NWS;
    uint64_t* b_full = w_empty + NWS;
    uint64_t* b_empty = b_full + NBS;
    uint64_t* acc_full = b_empty + NBS;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;         // abort path: completion of every issued MMA
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NXS; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], kSketchWarps / F::TEAMS); }
        for (int i = 0; i < NWS; ++i) { ptx::mbar_init(&w_full[i], 1); ptx::mbar_init(&w_empty[i], 1); }
        for (int i = 0; i < NBS; ++i) { ptx::mbar_init(&b_full[i], kSketchWarps / F::TEAMS); ptx::mbar_init(&b_empty[i], 1); }
        ptx::mbar_init(acc_full, 1);
        ptx::mbar_init(acc_empty, kEpiWarps);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 2) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) ptx::prefetch_tmap(&tmap_x);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tm = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------------ X loads (TMA)
        // One TMA instruction moves a [256 rows x 64 inputs] box (32 KB). The engine takes a
        // roughly fixed time per instruction, so boxes are as large as the layout allows.
        if (lane == 0) {
            int xp = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile / NB) * kRows;
                for (int kc = 0; kc < KC && ok; ++kc)
                    for (int p = 0; p < F::XPH; ++p, ++xp) {
                        const int slot = xp % NXS;
                        if (!ptx::mbar_wait(&x_empty[slot], ((xp / NXS) & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; report(status, abort_flag, 1); break; }
                        ptx::mbar_arrive_expect_tx(&x_full[slot], kXSlot);
                        ptx::tma_load_2d(xring + slot * kXSlot, &tmap_x, &x_full[slot], kc * BK + 64 * p, m0);
                    }
            }
            if (*abort_flag) drain_ring(x_full, NXS, xp, NXS);   // every issued copy lands before exit
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ Wc loads (cp.async)
        // Wc panels take the LSU path (16-byte cp.async per lane) so that the TMA engine serves X
        // only. A panel is published after the warp's copies land (wait_group) and a proxy fence.
        int wp = 0, pending = -1;
        bool ok = true;
        auto publish = [&](int i) {
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&w_full[i % NWS]);
        };
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int nb = tile % NB;
            for (int kc = 0; kc < KC && ok; ++kc)
                for (int sp = 0; sp < NSP; ++sp, ++wp) {
                    const int wi = wp % NWS;
                    if (!warp_wait(&w_empty[wi], ((wp / NWS) & 1) ^ 1, abort_flag)) { ok = false; if (lane == 0) report(status, abort_flag, 2); break; }
                    uint8_t* dst = wring + wi * F::W_PANEL;
                    const __nv_bfloat16* src = Wc + (size_t)nb * kNeu * Kc + (size_t)kc * S + sp * SP;
                    constexpr int kPieces = F::W_PANEL / 16, kPerRow = F::RB / 16;
#pragma unroll 4
                    for (int i = lane; i < kPieces; i += 32) {
                        const int r = i / kPerRow, c = i % kPerRow;
                        if (SS1_SPAN_IN(src + (size_t)r * Kc + c * 8 - Wc, 8, (int64_t)N * Kc, kSiteTc2Wc))
                            ptx::cp_async_16(dst + kmajor_off<F::RB>(r, c * 8), src + (size_t)r * Kc + c * 8);
                    }
                    asm volatile("cp.async.commit_group;" ::: "memory");
                    if (pending >= 0) {   // the previous panel's copies have landed
                        asm volatile("cp.async.wait_group 1;" ::: "memory");
                        publish(pending);
                    }
                    pending = wp;
                }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        if (ok && pending >= 0) publish(pending);
    } else if (warp == 2) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kNeu, kRows);
            int wc = 0;
            bool ok = true;
            for (int t = 0; t < my_tiles && ok; ++t) {
                // the epilogue must have read the previous tile's accumulator
                if (!ptx::mbar_wait(acc_empty, (t & 1) ^ 1, abort_flag, kWaitNs)) { ok = false; report(status, abort_flag, 3); break; }
                ptx::tc_fence_after();
                for (int kc = 0; kc < KC && ok; ++kc) {
                    for (int sp = 0; sp < NSP; ++sp, ++wc) {
                        const int wi = wc % NWS, bi = wc % NBS;
                        if (!ptx::mbar_wait(&w_full[wi], (wc / NWS) & 1, abort_flag, kWaitNs) ||
                            !ptx::mbar_wait(&b_full[bi], (wc / NBS) & 1, abort_flag, kWaitNs)) {
                            ok = false;
                            report(status, abort_flag, 4);
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t a0 = ptx::smem_u32(wring + wi * F::W_PANEL);
                        const uint32_t b0 = ptx::smem_u32(bring + bi * F::B_PANEL);
#pragma unroll
                        for (int kk = 0; kk < SP / 16; ++kk)
                            ptx::umma_bf16_ss(tm, ptx::smem_desc(a0 + kk * 32, 16, F::SBO, F::LAYOUT),
                                              ptx::smem_desc(b0 + kk * 32, 16, F::SBO, F::LAYOUT), idesc,
                                              (kc > 0 || sp > 0 || kk > 0) ? 1u : 0u);
                        ptx::umma_commit(&w_empty[wi]);
                        ptx::umma_commit(&b_empty[bi]);
                    }
                }
                if (ok) ptx::umma_commit(acc_full);
            }
            if (*abort_flag) {   // MMAs in flight finish before TMEM is released
                volatile int no_abort = 0;
                ptx::umma_commit(drain);
                ptx::mbar_wait(drain, 0, &no_abort, kWaitNs);
            }
        }
    } else if (warp < kFirstEpi) {
        // ------------------------------------------------------------------ sketch warps
        // A thread owns row r = 32*quad + lane (its TMEM lane) and row r + 128 of the tile.
        const int sw = warp - kFirstSketch;     // 0..15
        const int group = sw >> 2;              // k quarter of each staged box, slot quarter of each B panel
        const int quad = warp & 3;              // TMEM lanes 32*quad .. +31
        const int row0 = quad * 32 + lane;
        const uint32_t lane_base = tm + ((uint32_t)(quad * 32) << 16);
        const int G = my_tiles * KC;
        // Teams: with two TMEM staging buffers the 16 warps form two teams of 8 that take
        // alternate chunks, each with its own buffer, B slot and named barrier, so that one
        // team's staging (shared-memory reads) overlaps the other's gathering (TMEM reads).
        // With one buffer all 16 warps form one team.
        constexpr int kTeams = F::TEAMS, kTeamWarps = kSketchWarps / kTeams, kGroups = kTeamWarps / 4;
        const int team = sw / kTeamWarps;
        const int tgroup = (sw % kTeamWarps) >> 2;   // input part of each staged box, slot part of each panel
        const int bar_id = 2 + team;
        // Every warp of a team takes every named barrier of each of the team's chunks, also
        // after a time-out (then it only skips the work), so no partner can be left waiting.
        bool dead = false;
        // Stage chunk g into TMEM buffer xb as row pairs (X[r][k], X[r+128][k]) at column k.
        // This warp copies 64 / kGroups inputs of each box; the tcgen05.st stay in flight.
        auto stage = [&](int g, int xb) {
            constexpr int kIn = 64 / kGroups;        // inputs of a box per warp (16 or 32)
            const uint32_t xcol = kAccCols + (uint32_t)(xb * BK);
            for (int p = 0; p < F::XPH && !dead; ++p) {
                const int xp = g * F::XPH + p, slot = xp % NXS;
                if (!warp_wait(&x_full[slot], (xp / NXS) & 1, abort_flag)) {
                    dead = true;
                    if (lane == 0) report(status, abort_flag, 5);
                    break;
                }
                const uint8_t* p0 = xring + slot * kXSlot + row0 * 128;
                const uint8_t* p1 = p0 + 128 * 128;
                uint32_t v[kIn];
#pragma unroll
                for (int c = 0; c < kIn / 8; ++c) {   // 16-byte chunks (8 inputs each)
                    const uint32_t chunk = (uint32_t)(tgroup * (kIn / 8) + c) ^ (uint32_t)(row0 & 7);
                    const uint4 a = *reinterpret_cast<const uint4*>(p0 + chunk * 16);
                    const uint4 b = *reinterpret_cast<const uint4*>(p1 + chunk * 16);
                    v[8 * c + 0] = __byte_perm(a.x, b.x, 0x5410);
                    v[8 * c + 1] = __byte_perm(a.x, b.x, 0x7632);
                    v[8 * c + 2] = __byte_perm(a.y, b.y, 0x5410);
                    v[8 * c + 3] = __byte_perm(a.y, b.y, 0x7632);
                    v[8 * c + 4] = __byte_perm(a.z, b.z, 0x5410);
                    v[8 * c + 5] = __byte_perm(a.z, b.z, 0x7632);
                    v[8 * c + 6] = __byte_perm(a.w, b.w, 0x5410);
                    v[8 * c + 7] = __byte_perm(a.w, b.w, 0x7632);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&x_empty[slot]);
#pragma unroll
                for (int h = 0; h < kIn / 16; ++h)
                    ptx::tmem_st_32x32b_x16(lane_base + xcol + (uint32_t)(p * 64 + tgroup * kIn + 16 * h),
                                            *reinterpret_cast<const uint32_t(*)[16]>(v + 16 * h));
            }
        };
        // The team's stores of the staged chunk complete and become visible to its loads;
        // its loads issued before are ordered before any later store.
        auto team_barrier = [&](bool wait_st) {
            if (wait_st) ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::named_barrier_sync(bar_id, kTeamWarps * 32);
            ptx::tc_fence_after();
        };
        // Gather the sketch of chunk g (in TMEM buffer xb) into its B slots: one TMEM load
        // and one bf16x2 FMA per source give both rows' partial sums. A warp takes the
        // batches tgroup, tgroup + kGroups, ... of each panel for its 32 lanes; a load round
        // has kPerWarp batches' sources in flight before one wait.
        auto gather = [&](int g, int xb, const uint2* tab) {
            const uint32_t xaddr = lane_base + kAccCols + (uint32_t)(xb * BK);
            constexpr int kMyBatches = F::NBATCH / kGroups;   // batches of a panel per warp
            constexpr int kPerWarp = kMyBatches < 2 ? kMyBatches : 2;
            for (int sp = 0; sp < NSP; ++sp) {
                const int wc = g * NSP + sp, bi = wc % NBS;
                if (!warp_wait(&b_empty[bi], ((wc / NBS) & 1) ^ 1, abort_flag)) {
                    dead = true;
                    if (lane == 0) report(status, abort_flag, 6);
                    break;
                }
                uint8_t* bp = bring + bi * F::B_PANEL;
#pragma unroll 1
                for (int bt0 = tgroup; bt0 < F::NBATCH; bt0 += kGroups * kPerWarp) {
                    uint32_t w[kPerWarp][kBatch], m[kPerWarp][kBatch];
#pragma unroll
                    for (int u = 0; u < kPerWarp; ++u) {
                        const int e0 = (sp * SP + (bt0 + kGroups * u) * SB) * C;   // first source of batch u
#pragma unroll
                        for (int q = 0; q < kBatch / 2; ++q) {   // two {column, multiplier} entries per load
                            const uint4 e2 =
                                SS1_SPAN_IN(tab + e0 + 2 * q - gather_tab, 2, (int64_t)NB * KC * BK, kSiteTc2Tab)
                                    ? __ldg(reinterpret_cast<const uint4*>(tab + e0 + 2 * q))
                                    : make_uint4(0u, 0u, 0u, 0u);
                            w[u][2 * q] = ptx::tmem_ld_32x32b_x1(xaddr + e2.x);
                            m[u][2 * q] = e2.y;
                            w[u][2 * q + 1] = ptx::tmem_ld_32x32b_x1(xaddr + e2.z);
                            m[u][2 * q + 1] = e2.w;
                        }
                    }
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < kPerWarp; ++u) {
                        __nv_bfloat162 acc[SB];
#pragma unroll
                        for (int i = 0; i < SB; ++i) acc[i] = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
                        for (int idx = 0; idx < kBatch; ++idx)
                            acc[idx / C] = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&w[u][idx]),
                                                   *reinterpret_cast<const __nv_bfloat162*>(&m[u][idx]), acc[idx / C]);
                        uint32_t r0[SB / 2], r1[SB / 2];   // row r and row r + 128, slot pairs
#pragma unroll
                        for (int i = 0; i < SB / 2; ++i) {
                            const uint32_t x0 = *reinterpret_cast<uint32_t*>(&acc[2 * i]);
                            const uint32_t x1 = *reinterpret_cast<uint32_t*>(&acc[2 * i + 1]);
                            r0[i] = __byte_perm(x0, x1, 0x5410);
                            r1[i] = __byte_perm(x0, x1, 0x7632);
                        }
                        const int s0 = (bt0 + kGroups * u) * SB;   // first slot inside the panel
                        uint8_t* d0 = bp + kmajor_off<F::RB>(row0, s0);
                        uint8_t* d1 = bp + kmajor_off<F::RB>(row0 + 128, s0);
                        if constexpr (SB == 8) {
                            *reinterpret_cast<uint4*>(d0) = make_uint4(r0[0], r0[1], r0[2], r0[3]);
                            *reinterpret_cast<uint4*>(d1) = make_uint4(r1[0], r1[1], r1[2], r1[3]);
                        } else if constexpr (SB == 4) {
                            *reinterpret_cast<uint2*>(d0) = make_uint2(r0[0], r0[1]);
                            *reinterpret_cast<uint2*>(d1) = make_uint2(r1[0], r1[1]);
                        } else {
                            *reinterpret_cast<uint32_t*>(d0) = r0[0];
                            *reinterpret_cast<uint32_t*>(d1) = r1[0];
                        }
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&b_full[bi]);
            }
        };
        // Table of chunk g; the lines of this team's next chunk are pulled into L1 now, so that
        // its gathers do not wait for an L2 round trip before they can form TMEM addresses.
        auto table = [&](int g) -> const uint2* {
            const int tile = blockIdx.x + (g / KC) * gridDim.x, kc = g % KC;
            const int gn = g + kTeams, tn = blockIdx.x + (gn / KC) * gridDim.x, kn = gn % KC;
            if (gn < G) {
                const uint2* next = gather_tab + ((size_t)(tn % NB) * KC + kn) * BK;
                for (int sp = 0; sp < NSP; ++sp)
                    for (int bt = tgroup; bt < F::NBATCH; bt += kGroups)
                        if (lane == 0) asm volatile("prefetch.global.L1 [%0];" ::"l"(next + (sp * SP + bt * SB) * C));
            }
            return gather_tab + ((size_t)(tile % NB) * KC + kc) * BK;
        };
        for (int g = team; g < G; g += kTeams) {
            const int xb = kTeams == 2 ? team : 0;
            stage(g, xb);
            team_barrier(true);
            const uint2* tab = table(g);
            if (!dead) gather(g, xb, tab);
            team_barrier(false);   // this chunk's loads retire before the buffer is restaged
        }
    } else {
        // ------------------------------------------------------------------ epilogue warps
        // Warp `quad` owns neurons [32*quad, 32*quad + 32) of the tile. Per block of 32 rows:
        // 8 x tcgen05.ld.16x256b (mma fragment layout) -> bf16 -> stmatrix.trans into a private
        // [32 rows x 32 neurons] staging tile -> 16-byte coalesced stores of Y rows.
        const int quad = warp & 3;
        uint8_t* stg = estage + (warp - kFirstEpi) * kEpiStage;
        const int mi = lane >> 3, mj = lane & 7;
        int t = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
            const int nb = tile % NB, m0 = (tile / NB) * kRows;
            bool ok = warp_wait(acc_full, t & 1, abort_flag);
            if (!ok) { if (lane == 0) report(status, abort_flag, 7); break; }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int rb = 0; rb < kRows; rb += 32) {
                uint32_t r[4][8];
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const uint32_t col = (uint32_t)(rb + 8 * b);
                    ptx::tmem_ld_16x256b(tm + ((uint32_t)(quad * 32) << 16) + col, r[b][0], r[b][1], r[b][2], r[b][3]);
                    ptx::tmem_ld_16x256b(tm + ((uint32_t)(quad * 32 + 16) << 16) + col, r[b][4], r[b][5], r[b][6], r[b][7]);
                }
                ptx::tmem_ld_wait();
                if (rb == kRows - 32) {   // accumulator fully read: the next tile's MMAs may start
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(acc_empty);
                }
                // staging row y (0..31) holds neurons 0..31 as 64 bytes; 16-byte chunk c of row y
                // sits at chunk position c ^ ((y >> 1) & 3) so that both stmatrix and the reads
                // below touch distinct banks
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int y = 8 * b + mj;                      // staging row of this thread's address
                    const uint32_t off = (uint32_t)(y * 64) + ((uint32_t)(mi ^ ((y >> 1) & 3)) << 4);
                    ptx::stmatrix_x4_trans(ptx::smem_u32(stg + off), pack_bf16x2(r[b][0], r[b][1]), pack_bf16x2(r[b][2], r[b][3]),
                                           pack_bf16x2(r[b][4], r[b][5]), pack_bf16x2(r[b][6], r[b][7]));
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {   // 32 rows x 4 chunks = 128 pieces of 16 bytes
                    const int piece = i * 32 + lane, y = piece >> 2, c = piece & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(stg + y * 64 + ((c ^ ((y >> 1) & 3)) << 4));
                    const int m = m0 + rb + y;
                    if (m < M && SS1_SPAN_IN((size_t)m * N + (size_t)nb * kNeu + quad * 32 + c * 8, 8, (int64_t)M * N,
                                             kSiteTc2Y))
                        *reinterpret_cast<uint4*>(Y + (size_t)m * N + (size_t)nb * kNeu + quad * 32 + c * 8) = v;
                }
                __syncwarp();
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
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
    const cudaError_t attr_err = smem_attr_once(reinterpret_cast<const void*>(&tc2_kernel<BK, C>), F::SMEM);
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mx;
    if (!make_map(&mx, X, (uint64_t)L.K, (uint64_t)M, 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
    const int64_t mtiles = (M + kRows - 1) / kRows;
    const int64_t tiles = mtiles * L.NB;
    const int grid = (int)(tiles < L.num_sms ? tiles : L.num_sms);
    note_launch("tc2", (unsigned)grid, 1, 1, kThreads, F::SMEM, nullptr);
    tc2_kernel<BK, C><<<grid, kThreads, F::SMEM, st>>>(mx, (const __nv_bfloat16*)Wc, (__nv_bfloat16*)Y, L.d_gather, (int)M,
                                                       (int)L.N, (int)(L.K / L.c), L.KC, L.NB, (int)tiles, L.status_dev);
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
    if ((M + kRows - 1) / kRows * L.NB > (int64_t)1 << 30) return cudaErrorInvalidValue;
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
