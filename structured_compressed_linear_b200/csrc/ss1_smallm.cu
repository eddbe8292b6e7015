// Small-M SS1 forward (decode-sized batches, M <= 64 rows, bf16): stream Wc once at HBM rate.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": sketch the input by signed hashed additions, then multiply with the compressed
// weights. With a handful of rows the multiply is a matrix-vector product bound by reading Wc
// (N x K/c bf16), so this kernel is built around streaming Wc with many 16-byte loads in flight.
//
// Grid: x = groups of NPC = 4 G neurons (inside one N-block), y = groups of MT rows. For each
// segment of kSegC compressed columns (kSegC * c inputs) a CTA
//   1. issues the first Wc loads of the segment (they do not depend on the sketch),
//   2. sketches its rows for its N-block into shared memory, fp32:
//      Xs[m][j] = sum_t sign_t * X[m, chunk(j) * BK + k_t], gathering X through L1,
//   3. streams Wc: warp w owns 4 neurons (group w % G) and every (8 / G)-th run of 32 x 8
//      compressed columns (part w / G), 8 bf16 per lane per load with one load group in
//      flight ahead of the FMAs.
// The split of K across the warps of a group is reduced at the end in a fixed order through
// shared memory (deterministic), after a shuffle reduction across lanes; Y is rounded once.
// Every CTA of an N-block recomputes the block's sketch for its rows (L1/L2 reads of X beside
// the Wc stream). More than MT rows re-read Wc once per row group, from L2 when it fits there.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>

#include <mutex>

namespace ss1 {
namespace {

constexpr int kMaxRows = 64;             // largest M routed here
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSegC = 1024;              // compressed columns per segment (S divides it)

// The c source entries of one compressed column, loaded as one vector (c * 2 bytes, aligned).
template <int C>
__device__ __forceinline__ void load_entries(const uint16_t* e, uint16_t (&out)[C]) {
    if constexpr (C == 1) {
        out[0] = __ldg(e);
    } else if constexpr (C == 2) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(e));
        out[0] = (uint16_t)v;
        out[1] = (uint16_t)(v >> 16);
    } else if constexpr (C == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(e));
        out[0] = (uint16_t)v.x; out[1] = (uint16_t)(v.x >> 16);
        out[2] = (uint16_t)v.y; out[3] = (uint16_t)(v.y >> 16);
    } else {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(e));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = (uint16_t)w[i];
            out[2 * i + 1] = (uint16_t)(w[i] >> 16);
        }
    }
}

template <int MT, int G, int C>
__global__ void __launch_bounds__(kThreads) smallm_kernel(const __nv_bfloat16* __restrict__ X,
                                                          const __nv_bfloat16* __restrict__ Wc,
                                                          __nv_bfloat16* __restrict__ Y,
                                                          const uint16_t* __restrict__ src, int M, int K, int N,
                                                          int BN, int lgS, int KC) {
    constexpr int WPG = kWarps / G;      // warps sharing one group of 4 neurons
    constexpr int NPC = 4 * G;           // neurons per CTA
    __shared__ __align__(16) float xs[MT][kSegC];
    __shared__ float red[kWarps][4][MT];

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int grp = warp % G, part = warp / G;
    const int n0 = blockIdx.x * NPC;
    const int m0 = blockIdx.y * MT;
    const int rows = min(MT, M - m0);
    const int nb = n0 / BN;
    const int S = 1 << lgS, BK = S * C;
    const int Kc = K / C;
    const __nv_bfloat16* Xg = X + (size_t)m0 * K;
    const __nv_bfloat16* Wg = Wc + (size_t)(n0 + grp * 4) * Kc;
    const uint16_t* tab = src + (size_t)nb * KC * S * C;   // this block's entries, column-major order

    float acc[4][MT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[i][m] = 0.f;

    for (int j0 = 0; j0 < Kc; j0 += kSegC) {
        const int seg8 = min(kSegC, Kc - j0) / 8;    // 8-column groups in this segment
        // 1. first Wc loads of this segment
        int q = part * 32 + lane;
        uint4 wn[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            wn[i] = q < seg8 && SS1_SPAN_IN(Wg + (size_t)i * Kc + j0 + q * 8 - Wc, 8, (int64_t)N * Kc, kSiteSmallmWc)
                        ? __ldg(reinterpret_cast<const uint4*>(Wg + (size_t)i * Kc + j0 + q * 8))
                        : make_uint4(0, 0, 0, 0);
        // 2. sketch of this N-block for the segment
        for (int jj = threadIdx.x; jj < seg8 * 8; jj += kThreads) {
            const int j = j0 + jj;                                   // compressed column
            uint16_t e[C] = {};
            if (SS1_SPAN_IN(tab + (size_t)j * C - src, C, (int64_t)(N / BN) * K, kSiteSmallmTab))
                load_entries<C>(tab + (size_t)j * C, e);
            const __nv_bfloat16* xk = Xg + (size_t)(j >> lgS) * BK;  // its K-chunk
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= rows) break;
                float v = 0.f;
#pragma unroll
                for (int t = 0; t < C; ++t) {
                    const size_t xi = (size_t)m * K + (e[t] & kSrcIdxMask);
                    const float x = SS1_IN(xk + xi - X, (int64_t)M * K, kSiteSmallmX) ? __bfloat162float(xk[xi]) : 0.f;
                    v += (e[t] & kSrcNegBit) ? -x : x;
                }
                xs[m][jj] = v;
            }
        }
        __syncthreads();
        // 3. Wc stream against the sketch
        for (; q < seg8; q += 32 * WPG) {
            uint4 w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = wn[i];
            const int qn = q + 32 * WPG;
            if (qn < seg8) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    wn[i] = SS1_SPAN_IN(Wg + (size_t)i * Kc + j0 + qn * 8 - Wc, 8, (int64_t)N * Kc, kSiteSmallmWc)
                                ? __ldg(reinterpret_cast<const uint4*>(Wg + (size_t)i * Kc + j0 + qn * 8))
                                : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= rows) break;
                const float4 a = *reinterpret_cast<const float4*>(&xs[m][q * 8]);
                const float4 b = *reinterpret_cast<const float4*>(&xs[m][q * 8 + 4]);
                const float xv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w[i]);
                    float sacc = acc[i][m];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 wf = __bfloat1622float2(wp[t]);
                        sacc = fmaf(wf.x, xv[2 * t], sacc);
                        sacc = fmaf(wf.y, xv[2 * t + 1], sacc);
                    }
                    acc[i][m] = sacc;
                }
            }
        }
        __syncthreads();
    }
    // 4. lanes -> one value per (neuron, row) and warp; then the K parts in a fixed order
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = acc[i][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[i][m] = v;
        }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < MT; ++m) red[warp][i][m] = acc[i][m];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < rows * NPC; t += kThreads) {
        const int m = t / NPC, nl = t % NPC;
        float v = 0.f;
#pragma unroll
        for (int p = 0; p < WPG; ++p) v += red[p * G + nl / 4][nl % 4][m];
        const size_t yi = (size_t)(m0 + m) * N + n0 + nl;
        if (SS1_IN(yi, (int64_t)M * N, kSiteSmallmY)) Y[yi] = __float2bfloat16_rn(v);
    }
}

int log2_exact(int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return (1 << l) == v ? l : -1;
}

template <int MT, int G, int C>
cudaError_t launch_tpl(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    const dim3 grid((unsigned)(L.N / (4 * G)), (unsigned)((M + MT - 1) / MT));
    note_launch("smallm", grid.x, grid.y, 1, kThreads, 0, nullptr);
    smallm_kernel<MT, G, C><<<grid, kThreads, 0, st>>>((const __nv_bfloat16*)X, (const __nv_bfloat16*)Wc,
                                                       (__nv_bfloat16*)Y, L.d_src, (int)M, (int)L.K, (int)L.N,
                                                       L.BN, log2_exact(L.S), L.KC);
    return cudaGetLastError();
}

template <int MT, int G>
cudaError_t launch_c(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    switch (L.c) {
        case 1: return launch_tpl<MT, G, 1>(L, X, Wc, Y, M, st);
        case 2: return launch_tpl<MT, G, 2>(L, X, Wc, Y, M, st);
        case 4: return launch_tpl<MT, G, 4>(L, X, Wc, Y, M, st);
        default: return launch_tpl<MT, G, 8>(L, X, Wc, Y, M, st);
    }
}

template <int MT>
cudaError_t launch_rows(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    // widest neuron group that still gives every SM about four CTAs
    const int64_t row_groups = (M + MT - 1) / MT;
    const int64_t want = 4LL * L.num_sms;
    if (L.BN % 32 == 0 && (L.N / 32) * row_groups >= want) return launch_c<MT, 8>(L, X, Wc, Y, M, st);
    if (L.BN % 16 == 0 && (L.N / 16) * row_groups >= want) return launch_c<MT, 4>(L, X, Wc, Y, M, st);
    return launch_c<MT, 2>(L, X, Wc, Y, M, st);
}

}  // namespace

bool smallm_supported(const ss1_layer& L, int64_t M) {
    if (M < 1 || M > kMaxRows) return false;
    if (dec_supported(L, M)) return true;
    if (L.BN % 8 != 0) return false;
    const int lgS = log2_exact(L.S);
    if (lgS < 3 || (1 << lgS) > kSegC) return false;          // S a power of two in [8, kSegC]
    if (L.K % 8 != 0 || (L.K / L.c) % 8 != 0) return false;
    return true;
}

cudaError_t launch_smallm(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    if (dec_supported(L, M)) return launch_dec(L, X, Wc, Y, M, st);
    if (M <= 1) return launch_rows<1>(L, X, Wc, Y, M, st);
    if (M <= 2) return launch_rows<2>(L, X, Wc, Y, M, st);
    if (M <= 4) return launch_rows<4>(L, X, Wc, Y, M, st);
    return launch_rows<8>(L, X, Wc, Y, M, st);
}

}  // namespace ss1
