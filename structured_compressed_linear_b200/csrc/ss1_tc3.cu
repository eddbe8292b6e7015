// Tensor-core SS1 forward for sm_100a with the sketch itself computed by tcgen05.mma.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": the input is sketched (signed hashed additions shrink each K-chunk by the
// compression factor c) and the sketch is multiplied with the compressed weights. Per
// (N-block nb, K-chunk kc) the sketch is a linear map of the chunk,
//
//     Xs_nb[m, s] = sum_k X[m, k] * P_nb,kc[s, k],   P[s, k] = g_nb(k) if slot_nb(k) == s else 0,
//
// a 0/+-1 matrix with exactly one non-zero per input k. So the sketch is a small GEMM whose
// result is exact in the fp32 accumulator (c signed bf16 terms), rounded once to bf16. Both
// products run on the tensor cores; the CUDA cores only build P and convert the sketch.
//
// Tile: 128 rows of X (UMMA M) x Q N-blocks (Q = 2 for most shapes); one persistent CTA per SM
// takes tiles N-block-pair fastest. Per K-chunk:
//   * X-load warp  : X[m0:+128, chunk] as [128 x 64] TMA boxes (128B swizzle) into a ring.
//   * W-load warp  : the Q N-blocks' Wc[nb*128:+128, kc*S:+S] as TMA boxes into a ring of two
//                    chunks, or of three half chunks where that leaves room for one more X box.
//   * build warps  : one per (64-input unit, N-block) of a sketch segment (up to four). Each
//                    writes its unit's non-zeros into the stacked [Q*S x 64] K-major panel of
//                    the B operand (two entries per lane) and clears the previous use's entries,
//                    whose offsets it keeps in registers. Its table entries are loaded two
//                    segments ahead. The first N-block's warps also wait for their X box, and
//                    all of them raise sk_ready.
//   * sketch warp  : D_s[128 rows x Q*S] (fp32, TMEM, double-buffered) = X_chunk * P^T, BK/16
//                    UMMAs, one commit (seg_done) per segment; every consumer derives from that
//                    one barrier what it has freed.
//   * 8 convert warps (two per TMEM lane quarter, one per half of the sketch columns): fp32 ->
//                    bf16 in the A-operand layout (lane = row, two consecutive slots per 32-bit
//                    column), in place in D_s or into a separate buffer where TMEM has room. The
//                    first also waits for the chunk's Wc. All raise mm_ready.
//   * main warp    : D_j[128 rows x 128] += Xs_j (A operand from TMEM) * Wc_j^T, S/16 UMMAs per
//                    N-block j. At a tile's first chunk it waits per N-block for the epilogue to
//                    have read the accumulator. It commits the Wc stage and the sketch buffer
//                    back. Sketch and main products come from two warps, so that one warp's
//                    barrier waits overlap the other's UMMAs: a wait in the issuing thread drains
//                    the tensor pipe's short queue.
//   * 4 epilogue warps: accumulators -> bf16 (round to nearest even) -> swizzled shared-memory
//                    staging -> TMA bulk stores of [32 rows x 32 neurons] boxes (rows past M are
//                    clipped by the tensor map); each N-block's accumulator is released as soon
//                    as it has been read.
// Every mbarrier wait is bounded; a wait that runs out sets the CTA's abort flag and the
// handle's status word, drains the copies and MMAs in flight and returns (no trap).
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

namespace ss1 {

// defined in ss1_tc.cu (tensor-map encoding through the driver entry point)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

constexpr int kRows = 128;                 // rows of X per tile (UMMA M)
constexpr int kNeu = 128;                  // neurons per N-block (UMMA N of the main product)
constexpr int kUnitK = 64;                 // inputs per X box / sketch panel (one 128-byte swizzle row)
constexpr int kXUnit = kRows * 128;        // bytes of one X box [128 rows x 64 inputs]
constexpr int kWarpLoadX = 0, kWarpSketch = 1, kWarpBuild = 2, kWarpLoadW = 3, kFirstConv = 4, kConvWarps = 8;
constexpr int kFirstEpi = kFirstConv + kConvWarps, kEpiWarps = 4;
constexpr int kWarpMain = kFirstEpi + kEpiWarps;
constexpr int kFirstBuildExtra = kWarpMain + 1;   // further build warps (warp kWarpBuild is the first)
constexpr int kMaxBuildWarps = 4;
constexpr int kWarps = kFirstBuildExtra + kMaxBuildWarps - 1;
constexpr int kThreads = kWarps * 32;
constexpr int kEpiBox = 32 * 32 * 2;       // one [32 rows x 32 neurons] bf16 store box
constexpr int kSmemBudget = 225 * 1024;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint16_t kBf16One = 0x3F80u, kBf16MinusOne = 0xBF80u;

template <int BK, int C, int Q>
struct Cfg {
    static constexpr int S = BK / C;
    static constexpr int QS = Q * S;                     // N of the sketch UMMA
    static constexpr int HW = QS / 2;                    // sketch columns per convert warp
    static constexpr int U = BK / kUnitK;                // X boxes / sketch panels per chunk
    static constexpr int SU = U < 2 ? U : 2;             // units per sketch segment (one sk_ready)
    static constexpr int NSEG = U / SU;                  // segments per chunk
    static constexpr int P_UNIT = QS * 128;              // bytes of one sketch panel [QS x 64]
    static constexpr int RB = S >= 64 ? 128 : 2 * S;     // Wc operand: bytes per row of a panel
    static constexpr uint32_t WLAYOUT = S >= 64 ? ptx::kLayoutSW128 : (S == 32 ? ptx::kLayoutSW64 : ptx::kLayoutSW32);
    static constexpr int WSBO = 8 * RB;
    static constexpr int W_PANEL = kNeu * RB;            // bytes of one Wc panel
    static constexpr int W_NB = kNeu * S * 2;            // one N-block's Wc chunk
    static constexpr int W_STAGE = Q * W_NB;
    static constexpr int NP = 2 * SU;                    // sketch panels: two segments
    static constexpr int NBW = SU * Q;                   // build warps in use: one per (unit, N-block)
    static constexpr int EPI = kEpiWarps * 2 * kEpiBox;
    static constexpr int CLR = 0;
    // The Wc ring holds two chunks, or, where that frees room for one more X box, three half
    // chunks (a chunk's Wc panels in two halves, WH = 2): NWS slots of WU bytes, WH per chunk.
    static constexpr int WPAN = Q * ((S + 63) / 64);     // Wc panels per chunk
    static constexpr int NX_WHOLE = (kSmemBudget - NP * P_UNIT - 2 * W_STAGE - EPI - CLR) / kXUnit;
    static constexpr int NX_HALF = (kSmemBudget - NP * P_UNIT - 3 * (W_STAGE / 2) - EPI - CLR) / kXUnit;
    static constexpr int WH = (WPAN % 2 == 0 && NX_WHOLE < 2 * U + 1 && NX_HALF > NX_WHOLE) ? 2 : 1;
    static constexpr int WU = W_STAGE / WH;
    static constexpr int NW = WH == 2 ? 3 : 2;           // Wc ring slots
    static constexpr int FIXED = NP * P_UNIT + NW * WU + EPI + CLR;
    static constexpr int NX_FIT = (kSmemBudget - FIXED) / kXUnit;
    static constexpr int NX = NX_FIT < 2 * U + 1 ? NX_FIT : 2 * U + 1;
    // TMEM columns: Q accumulators (x NACC buffers), two fp32 sketch buffers D_s (QS columns each)
    // and, where the columns allow (SEP), two bf16 sketch buffers Xs (QS / 2 columns each, two
    // slots per column); otherwise the bf16 sketch is written inside its D_s buffer (in place).
    // Preference: two accumulators (the epilogue overlaps the next tile), then SEP.
    static constexpr int ACC_COLS = Q * kNeu;
    static constexpr int NACC = (2 * ACC_COLS + 2 * QS <= 512) ? 2 : 1;
    static constexpr bool SEP = NACC * ACC_COLS + 3 * QS <= 512;
    static constexpr int DS_COL = NACC * ACC_COLS;
    static constexpr int XS_COL = DS_COL + 2 * QS;
    // shared memory (the swizzled buffers first, each a multiple of 1 KB)
    static constexpr int OFF_X = 0;
    static constexpr int OFF_P = OFF_X + NX * kXUnit;
    static constexpr int OFF_W = OFF_P + NP * P_UNIT;
    static constexpr int OFF_E = OFF_W + NW * WU;
    static constexpr int OFF_TAB = OFF_E + EPI;
    static constexpr int OFF_CLR = OFF_TAB;
    static constexpr int OFF_BAR = OFF_CLR + CLR;
    static constexpr int NBAR = NX + 4 + 2 + 2 * NW + 2 + 2 + 2 + NACC + NACC * Q + 2 + 2;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    static_assert(BK % kUnitK == 0 && BK <= 256 && U % SU == 0, "chunks of whole 64-input units");
    static_assert(S % 16 == 0 && S >= 16 && S <= 128, "UMMA K-steps of 16 over the slots");
    static_assert(QS % 32 == 0 && QS <= 256 && HW % 16 == 0, "sketch UMMA N and conversion halves");
    static_assert(DS_COL + 2 * QS + (SEP ? QS : 0) <= 512, "TMEM budget");
    static_assert(NX >= 2 * SU && SMEM <= 227 * 1024, "shared memory budget: X ring holds two segments");
    static_assert(W_PANEL % 1024 == 0 && P_UNIT % 1024 == 0 && OFF_E % 1024 == 0 && WU % 1024 == 0,
                  "swizzle atoms stay aligned");
    static_assert(WH == 1 || W_NB == ((S + 63) / 64) * W_PANEL, "a chunk's panels lie back to back");
    static_assert(NBW <= kMaxBuildWarps, "build warps");
    // the X loader's first wait for segment g comes before the boxes of segment g + 4 are all
    // issued, so that segment (the same barrier, one phase later) cannot have completed yet
    static_assert(NX < 5 * SU, "X ring depth against the four segment barriers");
};

constexpr int kMaxLayers = 4;
enum { kActNone = 0, kActRelu = 1, kActGelu = 2 };

// One layer of a launch: its tensor maps (X [M x K], Wc [N x K/c], Y [M x N]), its slot table,
// and the epilogue's bias (bf16 [N], or null) and activation.
struct Tc3Layer {
    CUtensorMap tx, tw, ty;
    const uint16_t* slot_tab;
    const __nv_bfloat16* bias;
    int K, KC, NG, act;
};

// A launch runs one layer, its (M-tile, N-block group) tiles dealt round-robin to the CTAs, or
// (chain) up to kMaxLayers layers, each the input of the next: a CTA then takes pairs of M-tiles
// and carries both through every layer, alternating between them (layer l of tile A, layer l of
// tile B, layer l + 1 of A, ...), so no other CTA's output is ever waited for and the wait of one
// tile for its previous layer's stores is covered by the other tile's work.
struct Tc3Params {
    Tc3Layer layer[kMaxLayers];
    int n_layers;
    int chain;
    int num_units;   // tiles (one layer) or pairs of M-tiles (chain)
    int M;           // rows (a chain's pair may end in a tile wholly past M: its stores are skipped)
    int32_t* status;
    uint64_t wait_ns;       // limit of every wait (2 s; a test of the time-out path cuts it)
    int withhold_segment;   // test of the time-out path: CTA 0's first build warp skips this
                            // segment's arrival, so the sketch warp's wait runs out (-1: never)
};

struct TileInfo {
    int l, m0, nb0, ng, KC, h;   // h: which M-tile of the chain's pair (0 or 1)
};

// Tiles of one chain unit (a pair of M-tiles through all N-block groups of all layers) and their chunks.
__device__ __forceinline__ void chain_sizes(const Tc3Params& p, int& tiles, int& chunks) {
    tiles = 0;
    chunks = 0;
    for (int l = 0; l < p.n_layers; ++l) {
        tiles += 2 * p.layer[l].NG;
        chunks += 2 * p.layer[l].NG * p.layer[l].KC;
    }
}

// The j-th tile this CTA computes.
template <int Q, bool CHAIN>
__device__ __forceinline__ TileInfo tile_info(const Tc3Params& p, int j) {
    TileInfo t;
    if (!CHAIN) {
        const int tile = (int)blockIdx.x + j * (int)gridDim.x, NG = p.layer[0].NG;
        t.l = 0;
        t.h = 0;
        t.ng = tile % NG;
        t.m0 = (tile / NG) * kRows;
        t.KC = p.layer[0].KC;
    } else {
        int T, C;
        chain_sizes(p, T, C);
        int r = j % T, l = 0;
        while (l + 1 < p.n_layers && r >= 2 * p.layer[l].NG) r -= 2 * p.layer[l++].NG;
        t.l = l;
        t.h = r / p.layer[l].NG;
        t.ng = r % p.layer[l].NG;
        t.m0 = (2 * ((int)blockIdx.x + (j / T) * (int)gridDim.x) + t.h) * kRows;
        t.KC = p.layer[l].KC;
    }
    t.nb0 = t.ng * Q;
    return t;
}

// The i-th chunk this CTA processes: its tile and its K-chunk kc.
template <int Q, bool CHAIN>
__device__ __forceinline__ TileInfo chunk_info(const Tc3Params& p, int i, int& kc) {
    if (!CHAIN) {
        const int KC = p.layer[0].KC;
        kc = i % KC;
        return tile_info<Q, CHAIN>(p, i / KC);
    }
    int T, C;
    chain_sizes(p, T, C);
    int r = i % C, l = 0, j = (i / C) * T;
    while (l + 1 < p.n_layers && r >= 2 * p.layer[l].NG * p.layer[l].KC) {
        r -= 2 * p.layer[l].NG * p.layer[l].KC;
        j += 2 * p.layer[l++].NG;
    }
    kc = r % p.layer[l].KC;
    return tile_info<Q, CHAIN>(p, j + r / p.layer[l].KC);
}

__device__ __forceinline__ float activate(float v, int act) {
    if (act == kActRelu) return fmaxf(v, 0.0f);
    if (act == kActGelu) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));   // v * Phi(v)
    return v;
}

// The first wait of the CTA to run out writes its site; the warps it stalls then see the abort
// flag, give up their own waits and leave the word as it is. (Two waits that run out in the same
// instant may both write; either site is a true one.)
__device__ __forceinline__ void report(int32_t* status, volatile int* abort_flag, int site) {
    if (*abort_flag == 0) {
        *abort_flag = 1;
        *(volatile int32_t*)status = (kStatusKernelTC << 8) | (0x80 + site);
        __threadfence_system();
    }
}

// Lane 0 waits, the warp follows: one poller per warp instead of 32.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort_flag,
                                          uint64_t limit_ns) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, abort_flag, limit_ns);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Wait of an MMA-issuing warp: every lane polls the barrier without suspending (one shared-memory
// broadcast per poll), so the issue resumes as soon as the phase completes.
__device__ __forceinline__ bool warp_wait_spin(uint64_t* bar, uint32_t parity, const volatile int* abort_flag,
                                               uint64_t limit_ns) {
    bool ok = ptx::mbar_test(bar, parity);
    if (!ok) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (uint32_t n = 1;; ++n) {
            if (ptx::mbar_test(bar, parity)) { ok = true; break; }
            if ((n & 63) == 0 && (*abort_flag || ptx::globaltimer_ns() - t0 > limit_ns)) break;
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// Slot and phase of a ring position, advanced without divisions.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    int n;
    __device__ explicit Ring(int n_) : n(n_) {}
    __device__ __forceinline__ void next() {
        if (++slot == n) { slot = 0; phase ^= 1u; }
    }
};

// Waits for the last `depth` completions of a ring of `n` full-barriers after `issued` fills
// (used only to drain copies in flight after an abort).
__device__ __forceinline__ void drain_ring(uint64_t* full, int n, int issued, int depth) {
    volatile int no_abort = 0;
    for (int i = (issued - depth > 0 ? issued - depth : 0); i < issued; ++i)
        ptx::mbar_wait(&full[i % n], (uint32_t)((i / n) & 1), &no_abort, kWaitNs);
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo_f32, uint32_t hi_f32) {
    __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(lo_f32), __uint_as_float(hi_f32));
    return *reinterpret_cast<uint32_t*>(&b);
}

// Byte offset of element (row, kl) of a K-major [rows x 64] panel with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_off(int row, int kl) {
    return (uint32_t)(row * 128) + ((uint32_t)((kl >> 3) ^ (row & 7)) << 4) + (uint32_t)(kl & 7) * 2u;
}

// TEST: the variant for the test of the time-out path (runtime wait limit, one withheld arrival);
// the hot variants keep both out of their loops.
template <int BK, int C, int Q, bool CHAIN, bool FX, bool TEST>
__global__ void __launch_bounds__(kThreads, 1) tc3_kernel(const __grid_constant__ Tc3Params p) {
    using F = Cfg<BK, C, Q>;
    int32_t* status = p.status;
    const uint64_t wait_ns = TEST ? p.wait_ns : kWaitNs;
    constexpr int S = F::S, QS = F::QS, HW = F::HW, U = F::U, SU = F::SU, NSEG = F::NSEG;
    constexpr int NX = F::NX, NP = F::NP, NW = F::NW, NACC = F::NACC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xring = smem + F::OFF_X;
    uint8_t* pring = smem + F::OFF_P;
    uint8_t* wring = smem + F::OFF_W;
    uint8_t* estage = smem + F::OFF_E;
    // One tcgen05.commit per sketch segment (seg_done) tells every consumer at once: the X
    // loader and the build warp that the segment's X boxes and panels are free, the convert
    // warps (at a chunk's last segment) that the sketch is in D_s. Commits from the issuing
    // thread are kept few because each one costs about as much as a short UMMA.
    uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + F::OFF_BAR);
    uint64_t* seg_done = x_full + NX;     // [4] sketch segment g completed (g % 4)
    uint64_t* sk_ready = seg_done + 4;    // [2] panels + X boxes of a sketch segment ready
    uint64_t* w_full = sk_ready + 2;
    uint64_t* w_empty = w_full + NW;
    uint64_t* mm_ready = w_empty + NW;    // [2] Xs[b] written, Wc (and the accumulator) ready
    uint64_t* ds_free = mm_ready + 2;     // [2] D_s[b] may take the next sketch: SEP, the convert warps
                                          // have read it; in place, the main product has read its Xs
    uint64_t* xs_free = ds_free + 2;      // [2] (SEP) the main product has read Xs[b]
    uint64_t* acc_full = xs_free + 2;     // [NACC]
    uint64_t* acc_empty = acc_full + NACC;   // [NACC][Q] the epilogue has read N-block j's columns
    uint64_t* drain = acc_empty + NACC * Q;  // [2] abort path: completion of every MMA a warp issued
    uint64_t* layer_done = drain + 2;        // [2] chain: M-tile h of the pair has its layer stored
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(layer_done + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int my_units = (p.num_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    int my_tiles, G;   // tiles and chunks this CTA processes
    if (CHAIN) {
        int T, Cm;
        chain_sizes(p, T, Cm);
        my_tiles = my_units * T;
        G = my_units * Cm;
    } else {
        my_tiles = my_units;
        G = my_units * p.layer[0].KC;
    }

    // the sketch panels start zeroed; only their non-zeros are ever written afterwards
    for (int i = threadIdx.x; i < NP * F::P_UNIT / 16; i += kThreads)
        reinterpret_cast<uint4*>(pring)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        for (int i = 0; i < NX; ++i) ptx::mbar_init(&x_full[i], 1);
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&seg_done[i], 1);
        for (int i = 0; i < NW; ++i) { ptx::mbar_init(&w_full[i], 1); ptx::mbar_init(&w_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&sk_ready[i], F::NBW);
            ptx::mbar_init(&mm_ready[i], kConvWarps);
            ptx::mbar_init(&ds_free[i], F::SEP ? kConvWarps : 1);
            ptx::mbar_init(&xs_free[i], 1);
            ptx::mbar_init(&drain[i], 1);
        }
        for (int i = 0; i < NACC; ++i) ptx::mbar_init(&acc_full[i], 1);
        for (int i = 0; i < NACC * Q; ++i) ptx::mbar_init(&acc_empty[i], kEpiWarps);
        ptx::mbar_init(&layer_done[0], kEpiWarps);
        ptx::mbar_init(&layer_done[1], kEpiWarps);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpSketch) {
        ptx::tmem_alloc(tmem_slot, 512);
        ptx::tmem_relinquish();
    }
    if (lane == 0 && (warp == kWarpLoadX || warp == kWarpLoadW || warp == kFirstEpi)) {
        for (int l = 0; l < p.n_layers; ++l)
            ptx::prefetch_tmap(warp == kWarpLoadX ? &p.layer[l].tx : warp == kWarpLoadW ? &p.layer[l].tw : &p.layer[l].ty);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tm = *tmem_slot;

    if (warp == kWarpLoadX) {
        // ------------------------------------------------------------------ TMA loads of X
        if (lane == 0) {
            // A slot is free once the segment that read its previous box has completed. Segments
            // complete in order, so each is waited for once (seen = the latest observed): waiting
            // again on an old segment could read the barrier a full phase later and block (after
            // the long stall at a layer boundary, say, when every earlier segment is done).
            Ring xr(NX);
            int nx = 0, seen = -1;
            int layer_waits[2] = {0, 0};
            bool ok = true;
            for (int t = 0; t < my_tiles && ok; ++t) {
                const TileInfo ti = tile_info<Q, CHAIN>(p, t);
                if (CHAIN && ti.l > 0 && ti.ng == 0) {
                    // the M-tile's previous layer (this layer's X) has been stored by the epilogue
                    if (!ptx::mbar_wait(&layer_done[ti.h], (uint32_t)(layer_waits[ti.h] & 1), abort_flag, wait_ns)) {
                        report(status, abort_flag, 12);
                        break;
                    }
                    ++layer_waits[ti.h];
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                const CUtensorMap* tx = &p.layer[ti.l].tx;
                for (int kc = 0; kc < ti.KC && ok; ++kc)
                    for (int u = 0; u < U; ++u) {
                        if (nx >= NX) {   // the slot's previous unit belongs to segment gp
                            const int gp = (nx - NX) / SU;
                            if (gp > seen) {
                                if (!ptx::mbar_wait(&seg_done[gp & 3], (uint32_t)((gp >> 2) & 1), abort_flag, wait_ns)) { ok = false; report(status, abort_flag, 1); break; }
                                seen = gp;
                            }
                        }
                        ptx::mbar_arrive_expect_tx(&x_full[xr.slot], kXUnit);
                        ptx::tma_load_2d(xring + xr.slot * kXUnit, tx, &x_full[xr.slot], kc * BK + u * kUnitK, ti.m0);
                        xr.next();
                        ++nx;
                    }
            }
            if (*abort_flag) drain_ring(x_full, NX, nx, NX);   // every issued copy lands before exit
        }
    } else if (warp == kWarpLoadW) {
        // ------------------------------------------------------------------ TMA loads of Wc
        if (lane == 0) {
            Ring wr(NW);
            int nw = 0;
            bool ok = true;
            constexpr int PN = (S + 63) / 64, PPU = F::WPAN / F::WH;   // panels per N-block, per slot
            for (int t = 0; t < my_tiles && ok; ++t) {
                const TileInfo ti = tile_info<Q, CHAIN>(p, t);
                const int nb0 = ti.nb0;
                const CUtensorMap* tw = &p.layer[ti.l].tw;
                for (int kc = 0; kc < ti.KC && ok; ++kc) {
                    if constexpr (F::WH == 1) {
                        if (!ptx::mbar_wait(&w_empty[wr.slot], wr.phase ^ 1u, abort_flag, wait_ns)) { ok = false; report(status, abort_flag, 2); break; }
                        ptx::mbar_arrive_expect_tx(&w_full[wr.slot], F::W_STAGE);
                        uint8_t* wdst = wring + wr.slot * F::W_STAGE;
#pragma unroll
                        for (int j = 0; j < Q; ++j)
#pragma unroll
                            for (int pn = 0; pn < PN; ++pn)
                                ptx::tma_load_2d(wdst + j * F::W_NB + pn * F::W_PANEL, tw, &w_full[wr.slot], kc * S + pn * 64,
                                                 (nb0 + j) * kNeu);
                        wr.next();
                        ++nw;
                    } else {
#pragma unroll
                        for (int h = 0; h < F::WH; ++h) {   // slot h of the chunk: panels h*PPU .. +PPU
                            if (!ptx::mbar_wait(&w_empty[wr.slot], wr.phase ^ 1u, abort_flag, wait_ns)) { ok = false; report(status, abort_flag, 2); break; }
                            ptx::mbar_arrive_expect_tx(&w_full[wr.slot], F::WU);
                            uint8_t* wdst = wring + wr.slot * F::WU;
#pragma unroll
                            for (int q = 0; q < PPU; ++q) {
                                const int pnl = h * PPU + q, j = pnl / PN, pn = pnl % PN;
                                ptx::tma_load_2d(wdst + q * F::W_PANEL, tw, &w_full[wr.slot], kc * S + pn * 64, (nb0 + j) * kNeu);
                            }
                            wr.next();
                            ++nw;
                        }
                    }
                }
            }
            if (*abort_flag) drain_ring(w_full, NW, nw, NW);
        }
    } else if (warp == kWarpSketch) {
        // ------------------------------------------------------------------ sketch products
        // D_s[i & 1][128 rows x QS] = X_chunk * P^T, one sk_ready wait per segment of SU units;
        // the chunk's first segment also waits until the buffer's previous chunk (i - 2) has
        // released it. The whole warp walks the schedule; lane 0 issues.
        constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kRows, QS);
        const uint64_t xdesc0 = ptx::smem_desc(ptx::smem_u32(xring), 16, 1024, ptx::kLayoutSW128);
        const uint64_t pdesc0 = ptx::smem_desc(ptx::smem_u32(pring), 16, 1024, ptx::kLayoutSW128);
        const bool leader = lane == 0;
        Ring xr(NX);
        int seg = 0;
        bool ok = true;
        for (int i = 0; i < G && ok; ++i) {
            const uint32_t ds = tm + (uint32_t)(F::DS_COL + (i & 1) * QS);
            for (int sg = 0; sg < NSEG; ++sg, ++seg) {
                if (!warp_wait_spin(&sk_ready[seg & 1], (uint32_t)((seg >> 1) & 1), abort_flag, wait_ns) ||
                    (sg == 0 && i >= 2 && !warp_wait_spin(&ds_free[i & 1], (uint32_t)(((i >> 1) & 1) ^ 1), abort_flag, wait_ns))) {
                    ok = false;
                    if (leader) report(status, abort_flag, 3);
                    break;
                }
                ptx::tc_fence_after();
                uint64_t xd[SU], pd[SU];
#pragma unroll
                for (int su = 0; su < SU; ++su) {
                    xd[su] = xdesc0 + (uint64_t)((xr.slot * kXUnit) >> 4);
                    pd[su] = pdesc0 + (uint64_t)((((seg & 1) * SU + su) * F::P_UNIT) >> 4);
                    xr.next();
                }
                if (leader) {
#pragma unroll
                    for (int su = 0; su < SU; ++su)
#pragma unroll
                        for (int kk = 0; kk < kUnitK / 16; ++kk)
                            ptx::umma_bf16_ss(ds, xd[su] + (uint64_t)(kk * 2), pd[su] + (uint64_t)(kk * 2), idesc_s,
                                              (sg > 0 || su > 0 || kk > 0) ? 1u : 0u);
                    ptx::umma_commit(&seg_done[seg & 3]);
                }
                __syncwarp();
            }
        }
        if (*abort_flag && leader) {   // MMAs in flight finish before TMEM is released
            volatile int no_abort = 0;
            ptx::umma_commit(&drain[0]);
            ptx::mbar_wait(&drain[0], 0, &no_abort, kWaitNs);
        }
        __syncwarp();
    } else if (warp == kWarpMain) {
        // ------------------------------------------------------------------ compressed products
        // D_j[128 rows x 128] += Xs_j (A operand from TMEM) * Wc_j^T for the tile's Q N-blocks;
        // one mm_ready wait per chunk. A second issuing warp, so that one warp's waits overlap
        // the other's MMAs in the tensor pipe.
        constexpr uint32_t idesc_m = ptx::idesc_bf16_f32(kRows, kNeu);
        const uint64_t wdesc0 = ptx::smem_desc(ptx::smem_u32(wring), 16, F::WSBO, F::WLAYOUT);
        const bool leader = lane == 0;
        Ring wr(NW);
        int t = 0, kc = 0;
        int KC = my_tiles > 0 ? tile_info<Q, CHAIN>(p, 0).KC : 1;
        for (int i = 0; i < G; ++i) {
            const int b = i & 1, a = NACC == 2 ? (t & 1) : 0;
            if (!warp_wait_spin(&mm_ready[b], (uint32_t)((i >> 1) & 1), abort_flag, wait_ns)) {
                if (leader) report(status, abort_flag, 4);
                break;
            }
            ptx::tc_fence_after();
            const uint32_t xs = tm + (uint32_t)(F::SEP ? F::XS_COL + b * (QS / 2) : F::DS_COL + b * QS);
            const uint32_t acc_par = (uint32_t)(((t / NACC) & 1) ^ 1);   // n-th use of buffer a waits use n-1
            const uint32_t acc = tm + (uint32_t)(a * F::ACC_COLS);
            // the chunk's Wc slots (WH of them, in ring order from wr) and their descriptors
            int wslot[2] = {wr.slot, wr.slot};
            if constexpr (F::WH == 2) {
                Ring wr1 = wr;
                wr1.next();
                wslot[1] = wr1.slot;
            }
            const uint64_t wdb[2] = {wdesc0 + (uint64_t)((wslot[0] * F::WU) >> 4),
                                     F::WH == 2 ? wdesc0 + (uint64_t)((wslot[1] * F::WU) >> 4) : 0ull};
            bool stalled = false;
            if (leader) {
#pragma unroll
                for (int j = 0; j < Q; ++j) {
                    // a tile's first chunk: N-block j's accumulator columns have been read out
                    if (kc == 0) {
                        if (!ptx::mbar_wait(&acc_empty[a * Q + j], acc_par, abort_flag, wait_ns)) {
                            report(status, abort_flag, 11);
                            stalled = true;
                            break;
                        }
                        ptx::tc_fence_after();
                    }
#pragma unroll
                    for (int kk = 0; kk < S / 16; ++kk) {
                        constexpr int per_panel = F::RB / 2;   // slots per Wc panel row
                        const uint32_t off = (uint32_t)(j * F::W_NB + ((kk * 16) / per_panel) * F::W_PANEL +
                                                        ((kk * 16) % per_panel) * 2);
                        const int h = F::WH == 1 ? 0 : (int)(off / F::WU);   // which of the chunk's slots
                        const uint64_t wd = wdb[h] + (uint64_t)((off - (uint32_t)(h * F::WU)) >> 4);
                        // slots s0 .. s0+15 in bf16: SEP, column s0 / 2 of Xs[b]; in place, inside
                        // the converting warp's half of D_s[b]
                        const int s0 = j * S + kk * 16;
                        const uint32_t acol = F::SEP ? (uint32_t)(s0 / 2) : (uint32_t)((s0 / HW) * HW + (s0 % HW) / 2);
                        ptx::umma_bf16_ts(acc + (uint32_t)(j * kNeu), xs + acol, wd, idesc_m, (kc > 0 || kk > 0) ? 1u : 0u);
                    }
                }
#pragma unroll
                for (int h = 0; h < F::WH; ++h) ptx::umma_commit(&w_empty[wslot[h]]);
                ptx::umma_commit(F::SEP ? &xs_free[b] : &ds_free[b]);
                if (kc == KC - 1) ptx::umma_commit(&acc_full[a]);
            }
            if (__shfl_sync(0xffffffffu, stalled ? 1 : 0, 0)) break;
#pragma unroll
            for (int h = 0; h < F::WH; ++h) wr.next();
            if (++kc == KC) {
                kc = 0;
                if (++t < my_tiles) KC = tile_info<Q, CHAIN>(p, t).KC;
            }
        }
        if (*abort_flag && leader) {
            volatile int no_abort = 0;
            ptx::umma_commit(&drain[1]);
            ptx::mbar_wait(&drain[1], 0, &no_abort, kWaitNs);
        }
        __syncwarp();
    } else if (warp == kWarpBuild || (warp >= kFirstBuildExtra && warp < kFirstBuildExtra + F::NBW - 1)) {
        // ------------------------------------------------------------------ sketch matrices
        // Panel u of chunk kc for the tile's N-blocks nb0 .. nb0+Q-1: entry (j*S + slot(k), k)
        // = sign(k) for the 64 inputs k of the unit; every other entry stays zero. Build warp
        // bw writes unit su = bw % SU of each segment for N-block j = bw / SU: inputs lane and
        // lane + 32. Shared memory is slow to reach while the tensor core streams operands from
        // it, so the work is split over NBW warps whose latency chains overlap, each keeping its
        // shared accesses to the stores themselves: its table entries are loaded from global
        // memory into registers two segments ahead, and the offsets to clear when a panel comes
        // round again stay in registers (segments alternate between two panel pairs). The warps
        // of the first N-block also wait for their unit's X box, so sk_ready (all NBW warps)
        // means the whole segment is ready.
        const int bw = warp == kWarpBuild ? 0 : warp - kFirstBuildExtra + 1;
        const int su = bw % SU, j = bw / SU;
        const int nseg = G * NSEG;
        auto fetch = [&](int g, uint32_t (&e)[2]) {   // table entries of (segment g, su, j)
            if (g < nseg) {
                const int pu = g * SU + su, i = pu / U, u = pu % U;
                int kc;
                const TileInfo ti = chunk_info<Q, CHAIN>(p, i, kc);
                const Tc3Layer& ly = p.layer[ti.l];
                const uint16_t* src = ly.slot_tab + (size_t)(ti.nb0 + j) * ly.K + (size_t)kc * BK + u * kUnitK;
                [[maybe_unused]] const int64_t tab_n = (int64_t)ly.NG * Q * ly.K;
                e[0] = SS1_IN(src + lane - ly.slot_tab, tab_n, kSiteTc3Tab) ? __ldg(src + lane) : 0u;
                e[1] = SS1_IN(src + lane + 32 - ly.slot_tab, tab_n, kSiteTc3Tab) ? __ldg(src + lane + 32) : 0u;
            }
        };
        bool ok = true;
        uint32_t held0[2], held1[2];   // offsets written into this warp's panel of pair 0 / 1
        uint32_t ent0[2], ent1[2];     // table entries of the next even / odd segment
        fetch(0, ent0);
        fetch(1, ent1);
        auto segment = [&](int g, uint32_t (&held)[2], uint32_t (&ent)[2]) {
            const uint32_t e0 = ent[0], e1 = ent[1];
            fetch(g + 2, ent);
            uint8_t* panel = pring + ((g & 1) * SU + su) * F::P_UNIT;
            if (g >= 2) {   // the pair's previous segment (g - 2) has been multiplied
                if (!warp_wait_spin(&seg_done[(g - 2) & 3], (uint32_t)(((g - 2) >> 2) & 1), abort_flag, wait_ns)) {
                    ok = false;
                    if (lane == 0) report(status, abort_flag, 5);
                    return;
                }
                *reinterpret_cast<uint16_t*>(panel + held[0]) = 0;
                *reinterpret_cast<uint16_t*>(panel + held[1]) = 0;
            }
            held[0] = sw128_off(j * S + (int)(e0 & kSrcIdxMask), lane);
            held[1] = sw128_off(j * S + (int)(e1 & kSrcIdxMask), lane + 32);
            *reinterpret_cast<uint16_t*>(panel + held[0]) = (e0 & kSrcNegBit) ? kBf16MinusOne : kBf16One;
            *reinterpret_cast<uint16_t*>(panel + held[1]) = (e1 & kSrcNegBit) ? kBf16MinusOne : kBf16One;
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (j == 0) {   // unit su of the segment: its X box has landed
                const int xu = g * SU + su;
                if (!warp_wait_spin(&x_full[xu % NX], (uint32_t)((xu / NX) & 1), abort_flag, wait_ns)) {
                    ok = false;
                    if (lane == 0) report(status, abort_flag, 8);
                    return;
                }
            }
            if (lane == 0 && !(TEST && g == p.withhold_segment && blockIdx.x == 0 && bw == 0)) ptx::mbar_arrive(&sk_ready[g & 1]);
        };
        for (int g = 0; g < nseg && ok; g += 2) {
            segment(g, held0, ent0);
            if (ok && g + 1 < nseg) segment(g + 1, held1, ent1);
        }
    } else if (warp >= kFirstConv && warp < kFirstConv + kConvWarps) {
        // ------------------------------------------------------------------ sketch conversion
        // Warp (quarter, half) reads fp32 sketch columns [half*HW, half*HW + HW) of D_s[b] for its
        // 32 lanes and rounds them to bf16 pairs. SEP: it releases D_s[b] (ds_free) as soon as the
        // loads are done and writes columns [half*HW/2, +HW/2) of Xs[b] once the main product of
        // chunk i - 2 has read them. In place: it writes columns [half*HW, +HW/2) of D_s[b], which
        // only it has read.
        const int quad = warp & 3, half = (warp - kFirstConv) >> 2;
        const uint32_t lanes = (uint32_t)(quad * 32) << 16;
        Ring wr(NW);
        for (int i = 0; i < G; ++i) {
            const int b = i & 1;
            const int gl = i * NSEG + NSEG - 1;   // the chunk's last sketch segment
            if (!warp_wait_spin(&seg_done[gl & 3], (uint32_t)((gl >> 2) & 1), abort_flag, wait_ns)) {
                if (lane == 0) report(status, abort_flag, 6);
                break;
            }
            ptx::tc_fence_after();
            const uint32_t src = tm + lanes + (uint32_t)(F::DS_COL + b * QS + half * HW);
            uint32_t r[HW];
#pragma unroll
            for (int c0 = 0; c0 < HW; c0 += 16) ptx::tmem_ld_32x32b_x16(src + (uint32_t)c0, r + c0);
            ptx::tmem_ld_wait();
            ptx::tmem_ld_fence_regs<HW>(r);
            if (F::SEP) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&ds_free[b]);
            }
#pragma unroll
            for (int p = 0; p < HW / 2; ++p) r[p] = pack_bf16x2(r[2 * p], r[2 * p + 1]);
            uint32_t dst = src;
            if (F::SEP) {
                if (i >= 2 && !warp_wait_spin(&xs_free[b], (uint32_t)(((i >> 1) & 1) ^ 1), abort_flag, wait_ns)) {
                    if (lane == 0) report(status, abort_flag, 10);
                    break;
                }
                ptx::tc_fence_after();
                dst = tm + lanes + (uint32_t)(F::XS_COL + b * (QS / 2) + half * (HW / 2));
            }
#pragma unroll
            for (int c = 0; c < HW / 2; c += 8) ptx::tmem_st_32x32b_x8(dst + (uint32_t)c, r + c);
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            // the first convert warp also waits for the chunk's Wc (its WH slots)
            bool w_ok = true;
            if constexpr (F::WH == 1) {
                w_ok = warp != kFirstConv || warp_wait_spin(&w_full[wr.slot], wr.phase, abort_flag, wait_ns);
                wr.next();
            } else {
#pragma unroll
                for (int h = 0; h < F::WH; ++h) {
                    if (warp == kFirstConv && w_ok && !warp_wait_spin(&w_full[wr.slot], wr.phase, abort_flag, wait_ns)) w_ok = false;
                    wr.next();
                }
            }
            if (!w_ok) {
                if (lane == 0) report(status, abort_flag, 9);
                break;
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&mm_ready[b]);
        }
    } else if (warp >= kFirstEpi && warp < kFirstEpi + kEpiWarps) {
        // ------------------------------------------------------------------ epilogue
        // Warp `quad` owns rows [32 quad, 32 quad + 32) of the tile. Per [32 x 32] block: two
        // blocks' TMEM loads in flight, bf16 rounding, a swizzled (64-byte) staging box, one TMA
        // store; two staging boxes alternate so that a store's read overlaps the next block.
        const int quad = warp & 3;
        uint8_t* stg = estage + (warp - kFirstEpi) * 2 * kEpiBox;
        const uint32_t lane_base = tm + ((uint32_t)(quad * 32) << 16);
        int nst = 0;
        for (int t = 0; t < my_tiles; ++t) {
            const TileInfo ti = tile_info<Q, CHAIN>(p, t);
            const Tc3Layer& ly = p.layer[ti.l];
            const CUtensorMap* ty = &ly.ty;
            const __nv_bfloat16* bias = ly.bias;
            const int act = ly.act;
            const int a = NACC == 2 ? (t & 1) : 0;
            if (!warp_wait(&acc_full[a], (uint32_t)((t / NACC) & 1), abort_flag, wait_ns)) {
                if (lane == 0) report(status, abort_flag, 7);
                break;
            }
            ptx::tc_fence_after();
            const int row0 = ti.m0 + quad * 32;
            const int col0 = ti.nb0 * kNeu;
            auto store_block = [&](int q, uint32_t (&r)[32]) {
                uint8_t* box = stg + (nst & 1) * kEpiBox;
                if constexpr (FX) {   // bias of column col0 + 32 q + j (lane j loads it), then the activation
                    const float bl = bias && SS1_IN(col0 + q * 32 + lane, (int64_t)ly.NG * Q * kNeu, kSiteTc3Bias)
                                         ? __bfloat162float(bias[col0 + q * 32 + lane])
                                         : 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        r[jj] = __float_as_uint(activate(__uint_as_float(r[jj]) + __shfl_sync(0xffffffffu, bl, jj), act));
                }
                if (lane == 0) ptx::tma_store_wait_read1();   // the store two blocks ago has read `box`
                __syncwarp();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    *reinterpret_cast<uint4*>(box + lane * 64 + ((ch ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(pack_bf16x2(r[8 * ch + 0], r[8 * ch + 1]), pack_bf16x2(r[8 * ch + 2], r[8 * ch + 3]),
                                   pack_bf16x2(r[8 * ch + 4], r[8 * ch + 5]), pack_bf16x2(r[8 * ch + 6], r[8 * ch + 7]));
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (row0 < p.M) ptx::tma_store_2d(ty, box, col0 + q * 32, row0);
                    ptx::tma_store_commit();
                }
                ++nst;
            };
            const uint32_t abase = lane_base + (uint32_t)(a * F::ACC_COLS);
            if constexpr (FX) {
                // with bias and activation: each block loaded, waited for, then processed, so that
                // no register an asynchronous TMEM load still writes is touched meanwhile
#pragma unroll 1
                for (int q = 0; q < 4 * Q; ++q) {
                    uint32_t r[32];
                    ptx::tmem_ld_32x32b_x32(abase + (uint32_t)(q * 32), r);
                    ptx::tmem_ld_wait();
                    ptx::tmem_ld_fence_regs<32>(r);
                    if ((q + 1) % 4 == 0) {   // N-block q / 4 read: the next tile's MMAs into it may start
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&acc_empty[a * Q + q / 4]);
                    }
                    store_block(q, r);
                }
            } else {
            // two register buffers: the next block's TMEM load is in flight while this block is
            // staged and stored; N-block j is released right after its last block (4j+3) has landed
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32x32b_x32(abase, ra);
            ptx::tmem_ld_wait();
            ptx::tmem_ld_fence_regs<32>(ra);
#pragma unroll 1
            for (int q = 0; q < 4 * Q; q += 2) {
                ptx::tmem_ld_32x32b_x32(abase + (uint32_t)((q + 1) * 32), rb);
                store_block(q, ra);
                ptx::tmem_ld_wait();
                ptx::tmem_ld_fence_regs<32>(rb);
                if ((q + 2) % 4 == 0) {   // N-block q / 4 read: the next tile's MMAs into it may start
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[a * Q + q / 4]);
                }
                if (q + 2 < 4 * Q) ptx::tmem_ld_32x32b_x32(abase + (uint32_t)((q + 2) * 32), ra);
                store_block(q + 1, rb);
                if (q + 2 < 4 * Q) {
                    ptx::tmem_ld_wait();
                    ptx::tmem_ld_fence_regs<32>(ra);
                }
            }
            }
            if (CHAIN && ti.l + 1 < p.n_layers && ti.ng == ly.NG - 1) {
                // this warp's rows of the M-tile's layer are stored; once all four warps say so
                // the next layer may load them (the stores complete before the arrival)
                if (lane == 0) {
                    ptx::tma_store_wait0();
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    __threadfence();
                    ptx::mbar_arrive(&layer_done[ti.h]);
                }
                __syncwarp();
            }
        }
        if (lane == 0) ptx::tma_store_wait0();
        __syncwarp();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kWarpSketch) {
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

// One layer of a launch, as the host describes it.
struct Tc3Job {
    const ss1_layer* L;
    const void* X;
    const void* Wc;
    void* Y;
    const void* bias;
    int act;
};

template <int BK, int C, int Q>
cudaError_t launch_cfg(const Tc3Job* jobs, int n, bool chain, int64_t M, uint64_t wait_ns, int withhold,
                       cudaStream_t st) {
    using F = Cfg<BK, C, Q>;
    constexpr int S = F::S;
    bool fx = chain;
    for (int l = 0; l < n; ++l) fx = fx || jobs[l].bias != nullptr || jobs[l].act != kActNone;
    const bool test = withhold >= 0;
    // the test variant exists for one configuration only (BK = 128, c = 2, two N-blocks per tile)
    constexpr bool kTestCfg = BK == 128 && C == 2 && Q == 2;
    if (test && (!kTestCfg || chain || fx)) return cudaErrorInvalidValue;
    // three variants: one layer without bias or activation, one layer with them, a chain (with them)
    const void* fn = chain ? reinterpret_cast<const void*>(&tc3_kernel<BK, C, Q, true, true, false>)
                     : fx  ? reinterpret_cast<const void*>(&tc3_kernel<BK, C, Q, false, true, false>)
                           : reinterpret_cast<const void*>(&tc3_kernel<BK, C, Q, false, false, false>);
    if constexpr (kTestCfg)
        if (test) fn = reinterpret_cast<const void*>(&tc3_kernel<BK, C, Q, false, false, true>);
    const cudaError_t attr_err = smem_attr_once(fn, F::SMEM);
    if (attr_err != cudaSuccess) return attr_err;
    Tc3Params prm;
    memset(&prm, 0, sizeof(prm));
    const CUtensorMapSwizzle wsw = S >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (S == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    for (int l = 0; l < n; ++l) {
        const ss1_layer& L = *jobs[l].L;
        Tc3Layer& ly = prm.layer[l];
        if (!make_map(&ly.tx, jobs[l].X, (uint64_t)L.K, (uint64_t)M, kUnitK, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&ly.tw, jobs[l].Wc, (uint64_t)(L.K / L.c), (uint64_t)L.N, S >= 64 ? 64 : S, kNeu, wsw) ||
            !make_map(&ly.ty, jobs[l].Y, (uint64_t)L.N, (uint64_t)M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
        ly.slot_tab = L.d_slot;
        ly.bias = static_cast<const __nv_bfloat16*>(jobs[l].bias);
        ly.K = (int)L.K;
        ly.KC = L.KC;
        ly.NG = L.NB / Q;
        ly.act = jobs[l].act;
    }
    prm.n_layers = n;
    prm.chain = chain ? 1 : 0;
    prm.status = jobs[0].L->status_dev;
    prm.wait_ns = wait_ns;
    prm.withhold_segment = withhold;
    const int64_t mtiles = (M + kRows - 1) / kRows;
    const int64_t units = chain ? (mtiles + 1) / 2 : mtiles * prm.layer[0].NG;   // chain: pairs of M-tiles
    const int sms = jobs[0].L->num_sms;
    prm.num_units = (int)units;
    prm.M = (int)M;
    const int grid = (int)(units < sms ? units : sms);
    note_launch("tc3", (unsigned)grid, 1, 1, kThreads, F::SMEM, nullptr);
    if (chain)
        tc3_kernel<BK, C, Q, true, true, false><<<grid, kThreads, F::SMEM, st>>>(prm);
    else if (fx)
        tc3_kernel<BK, C, Q, false, true, false><<<grid, kThreads, F::SMEM, st>>>(prm);
    else if constexpr (kTestCfg) {
        if (test)
            tc3_kernel<BK, C, Q, false, false, true><<<grid, kThreads, F::SMEM, st>>>(prm);
        else
            tc3_kernel<BK, C, Q, false, false, false><<<grid, kThreads, F::SMEM, st>>>(prm);
    } else {
        tc3_kernel<BK, C, Q, false, false, false><<<grid, kThreads, F::SMEM, st>>>(prm);
    }
    return cudaGetLastError();
}

// N-blocks per tile: two where the N-blocks pair up (the sketch UMMA then has N = 2 S), one
// for S = 128 (already N = 128) or an odd count of N-blocks.
int pick_q(const ss1_layer& L) {
    if (L.S == 128) return 1;
    return L.NB % 2 == 0 ? 2 : 1;
}

}  // namespace

bool tc3_supported(const ss1_layer& L) {
    if (L.BN != kNeu || L.c < 2) return false;
    if (!(L.BK == 128 || L.BK == 256)) return false;
    if (!(L.S == 16 || L.S == 32 || L.S == 64 || L.S == 128)) return false;
    if ((pick_q(L) * L.S) % 32 != 0) return false;
    if (L.K % 8 != 0 || (L.K / L.c) % 8 != 0 || L.N % 8 != 0) return false;
    return true;
}

namespace {

// Dispatch on (BK, c, Q) of the first layer; every layer of a chain has the same three.
cudaError_t launch_jobs(const Tc3Job* jobs, int n, bool chain, int64_t M, cudaStream_t st, uint64_t wait_ns = kWaitNs,
                        int withhold = -1) {
    const ss1_layer& L = *jobs[0].L;
    if ((M + kRows - 1) / kRows * L.NB > (int64_t)1 << 30) return cudaErrorInvalidValue;
    const int q = pick_q(L);
#define SS1_TC3_CASE(bk, cc, qq) \
    if (L.BK == bk && L.c == cc && q == qq) return launch_cfg<bk, cc, qq>(jobs, n, chain, M, wait_ns, withhold, st);
    SS1_TC3_CASE(128, 2, 2)
    SS1_TC3_CASE(128, 2, 1)
    SS1_TC3_CASE(128, 4, 2)
    SS1_TC3_CASE(128, 4, 1)
    SS1_TC3_CASE(128, 8, 2)
    SS1_TC3_CASE(256, 2, 1)
    SS1_TC3_CASE(256, 4, 2)
    SS1_TC3_CASE(256, 4, 1)
    SS1_TC3_CASE(256, 8, 2)
    SS1_TC3_CASE(256, 8, 1)
#undef SS1_TC3_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_tc3(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, const void* bias, int act,
                       cudaStream_t st) {
    const Tc3Job job{&L, X, Wc, Y, bias, act};
    return launch_jobs(&job, 1, false, M, st);
}

cudaError_t launch_tc3_withhold(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M,
                                uint64_t wait_ns, cudaStream_t st) {
    const Tc3Job job{&L, X, Wc, Y, nullptr, kActNone};
    return launch_jobs(&job, 1, false, M, st, wait_ns, 2);
}

bool tc3_chain_ok(const ss1_layer* const* Ls, int n) {
    if (n < 1 || n > kMaxLayers) return false;
    for (int l = 0; l < n; ++l) {
        if (!tc3_supported(*Ls[l])) return false;
        if (Ls[l]->BK != Ls[0]->BK || Ls[l]->c != Ls[0]->c || pick_q(*Ls[l]) != pick_q(*Ls[0])) return false;
        if (Ls[l]->device != Ls[0]->device) return false;
        if (l > 0 && Ls[l]->K != Ls[l - 1]->N) return false;
    }
    return true;
}

cudaError_t launch_tc3_chain(const ss1_layer* const* Ls, int n, const void* X, const void* const* Wc, void* const* Y,
                             const void* const* bias, const int* act, int64_t M, cudaStream_t st) {
    Tc3Job jobs[kMaxLayers];
    for (int l = 0; l < n; ++l) jobs[l] = Tc3Job{Ls[l], l == 0 ? X : Y[l - 1], Wc[l], Y[l], bias ? bias[l] : nullptr,
                                                 act ? act[l] : kActNone};
    return launch_jobs(jobs, n, true, M, st);
}

}  // namespace ss1
