// Dense -> SS1 projection: the compressed weights closest (least squares) to a dense weight.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Key results": pre-trained dense layers (BERT, Llama-3-8B) are projected onto SS1 and used
// with or without finetuning. The pages print no formula; the plainest reading is the
// orthogonal projection onto the tied weights. The tied weight of N-block nb is
// W_full_nb = Wc_nb P_nb, with P_nb[j, k] = g_nb(k) if h_nb(k) == j: every row of P_nb holds
// exactly c entries of +-1, so P P^T = c I and the Frobenius-closest Wc is
//
//     Wc[n, j] = (1 / c) * sum over k with h_nb(k) == j of g_nb(k) * W[n, k],   nb = n / BN.
//
// (With the factor 1 instead of 1 / c the same kernel gives the weight gradient's tied sum,
// dWc = sum over the slot's inputs of g * dW_full; see ss1_backward.cu.)
// That is the forward pass's sketch applied to the rows of W (one neuron per row) with the
// N-block of the neuron, scaled by 1 / c. The work is a gather: each output reads c inputs of
// its row. The kernel is bound by HBM (W read once, Wc written once).
//
// The work is one (N-block, K-chunk) of W at a time: the chunk's table of sources is the same for
// all BN rows of the N-block, so a CTA reads it once and keeps it in registers, and each warp
// streams rows of W through its own small shared-memory buffer, gathering from it.
//   * fp32: the row kernel, one row per buffer fill.
//   * bf16: the pair kernel, two rows interleaved per buffer fill (one 32-bit word holds the
//     same input of both rows), so each shared-memory load serves two outputs.
// Each output sums its c terms pairwise in fp32, times the factor, rounded once to the output
// type; the order of the sum is the same in both kernels.
// Shapes whose rows or chunks are not 16-byte multiples take a plain kernel: one thread per
// output, reading its c inputs from global memory.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>

namespace ss1 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Row kernel: a CTA takes one (N-block, K-chunk, row range) and its 8 warps take the range's
// rows in turn. The chunk's table (BK entries, slot-major) is read once per CTA: lane l keeps the
// sources of its slots l, l + 32, ... (S * C = BK <= 256, so at most 8 entries). Per row, a warp
// reads the row's chunk (BK elements) with 16-byte loads, kRowsAhead of its rows ahead of the one
// it gathers (4 KB in flight per warp), stores it into its own shared-memory row buffer, and
// each lane sums its slots' C signed terms (pairwise), scales and writes them: 32
// consecutive outputs per store instruction. The N-block's rows are split over several CTAs when
// the (N-block, K-chunk) pairs alone would leave SMs idle.

template <typename T, int C>
__global__ void __launch_bounds__(kThreads, 3)
    project_rows_kernel(const T* __restrict__ W, T* __restrict__ Wc, const uint16_t* __restrict__ src_tab, int K,
                        int BK, int BN, int KC, int rows_per_cta, float scale) {
    constexpr int E = (int)sizeof(T);
    constexpr int kMaxVec = 256 * E / 512;                  // 16-byte vectors per lane of a 256-input row
    constexpr int kRowsAhead = 8 / kMaxVec;
    constexpr int kSlots = 8 / C;                           // slots per lane at most (S <= 256 / C)
    __shared__ __align__(16) uint8_t rowbuf[kWarps][256 * E];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kc = blockIdx.x, nb = blockIdx.y;
    const int S = BK / C, Kc = K / C;
    const int nvec = BK * E / 16;                           // 16-byte vectors in a row's chunk
    uint16_t ent[kSlots * C];                               // slot lane + 32 k, term j: ent[k * C + j]
    const uint16_t* tab = src_tab + ((size_t)nb * KC + kc) * BK;
#pragma unroll
    for (int k = 0; k < kSlots; ++k)
#pragma unroll
        for (int j = 0; j < C; ++j) {
            const int sl = lane + 32 * k;
            ent[k * C + j] = sl < S && SS1_IN(tab + sl * C + j - src_tab, (int64_t)gridDim.y * KC * BK, kSiteProjTab)
                                 ? __ldg(tab + sl * C + j)
                                 : (uint16_t)0;
        }
    const int r_lo = blockIdx.z * rows_per_cta, r_hi = min(BN, r_lo + rows_per_cta);
    const T* wrow0 = W + ((size_t)nb * BN + r_lo) * K + (size_t)kc * BK;
    T* crow0 = Wc + ((size_t)nb * BN + r_lo) * Kc + (size_t)kc * S;
    const int rows = r_hi - r_lo;
    uint4 buf[kRowsAhead][kMaxVec];
    auto load = [&](int r, uint4 (&v)[kMaxVec]) {
        if (r < rows) {
#pragma unroll
            for (int q = 0; q < kMaxVec; ++q) {
                const int vi = lane + 32 * q;
                if (vi < nvec && SS1_SPAN_IN(wrow0 + (size_t)r * K + vi * (16 / E) - W, 16 / E,
                                             (int64_t)gridDim.y * BN * K, kSiteProjW))
                    v[q] = __ldg(reinterpret_cast<const uint4*>(wrow0 + (size_t)r * K) + vi);
            }
        }
    };
#pragma unroll
    for (int a = 0; a < kRowsAhead; ++a) load(warp + a * kWarps, buf[a]);
    uint8_t* rb = rowbuf[warp];
    const T* x = reinterpret_cast<const T*>(rb);
    for (int r0 = warp; r0 < rows; r0 += kRowsAhead * kWarps) {
#pragma unroll
        for (int a = 0; a < kRowsAhead; ++a) {
            const int r = r0 + a * kWarps;
            if (r >= rows) break;
#pragma unroll
            for (int q = 0; q < kMaxVec; ++q) {
                const int vi = lane + 32 * q;
                if (vi < nvec) reinterpret_cast<uint4*>(rb)[vi] = buf[a][q];
            }
            load(r + kRowsAhead * kWarps, buf[a]);   // in flight during this row's gather
            __syncwarp();
#pragma unroll
            for (int k = 0; k < kSlots; ++k) {
                const int sl = lane + 32 * k;
                if (sl < S) {
                    float t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        t[j] = 0.0f;
                        if (j < C) {
                            const uint16_t e = ent[k * C + j];
                            const float v = (float)x[e & kSrcIdxMask];
                            t[j] = (e & kSrcNegBit) ? -v : v;
                        }
                    }
#pragma unroll
                    for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
                        for (int j = 0; j < w2; ++j) t[j] += t[j + w2];
                    if (SS1_IN(crow0 + (size_t)r * Kc + sl - Wc, (int64_t)gridDim.y * BN * Kc, kSiteProjWc))
                        crow0[(size_t)r * Kc + sl] = (T)(t[0] * scale);
                }
            }
            __syncwarp();
        }
    }
}

// bf16 pair kernel: the row kernel with two rows (r, r + 8) gathered at once. Their chunks are
// interleaved in the warp's buffer, one 32-bit word holding input k of both rows, so one
// shared-memory load serves both rows' terms: half the gathers of the row kernel, which is bound
// by them. The interleaved store writes, from lanes 0-3 and 4-7 of each quarter warp, the two
// halves of a lane's 32 bytes in opposite order, so the 8 lanes of a phase cover all 32 banks.
template <int C>
__global__ void __launch_bounds__(kThreads, 3)
    project_pairs_kernel(const __nv_bfloat16* __restrict__ W, __nv_bfloat16* __restrict__ Wc,
                         const uint16_t* __restrict__ src_tab, int K, int BK, int BN, int KC, int rows_per_cta,
                         float scale) {
    constexpr int kPairsAhead = 4;                          // 8 rows of 512 bytes in flight per warp
    constexpr int kSlots = 8 / C;
    __shared__ __align__(16) uint32_t pairbuf[kWarps][256];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kc = blockIdx.x, nb = blockIdx.y;
    const int S = BK / C, Kc = K / C;
    const int nvec = BK / 8;                                // 16-byte vectors in a row's chunk
    uint16_t ent[kSlots * C];
    const uint16_t* tab = src_tab + ((size_t)nb * KC + kc) * BK;
#pragma unroll
    for (int k = 0; k < kSlots; ++k)
#pragma unroll
        for (int j = 0; j < C; ++j) {
            const int sl = lane + 32 * k;
            ent[k * C + j] = sl < S && SS1_IN(tab + sl * C + j - src_tab, (int64_t)gridDim.y * KC * BK, kSiteProjTab)
                                 ? __ldg(tab + sl * C + j)
                                 : (uint16_t)0;
        }
    const int r_lo = blockIdx.z * rows_per_cta, r_hi = min(BN, r_lo + rows_per_cta);
    const __nv_bfloat16* wrow0 = W + ((size_t)nb * BN + r_lo) * K + (size_t)kc * BK;
    __nv_bfloat16* crow0 = Wc + ((size_t)nb * BN + r_lo) * Kc + (size_t)kc * S;
    const int rows = r_hi - r_lo;
    // pair p of this warp: rows warp + 16 p and warp + 16 p + 8
    uint4 buf[kPairsAhead][2];
    auto load = [&](int p, uint4 (&v)[2]) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = warp + 16 * p + 8 * i;
            v[i] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows && lane < nvec &&
                SS1_SPAN_IN(wrow0 + (size_t)r * K + lane * 8 - W, 8, (int64_t)gridDim.y * BN * K, kSiteProjW))
                v[i] = __ldg(reinterpret_cast<const uint4*>(wrow0 + (size_t)r * K) + lane);
        }
    };
#pragma unroll
    for (int a = 0; a < kPairsAhead; ++a) load(a, buf[a]);
    uint32_t* pb = pairbuf[warp];
    const int sw = (lane >> 2) & 1;
    for (int p0 = 0; warp + 16 * p0 < rows; p0 += kPairsAhead) {
#pragma unroll
        for (int a = 0; a < kPairsAhead; ++a) {
            const int p = p0 + a;
            const int ra = warp + 16 * p, rb = ra + 8;
            if (ra >= rows) break;
            if (lane < nvec) {
                const uint4 u = buf[a][0], v = buf[a][1];
                const uint4 lo = make_uint4(__byte_perm(u.x, v.x, 0x5410), __byte_perm(u.x, v.x, 0x7632),
                                            __byte_perm(u.y, v.y, 0x5410), __byte_perm(u.y, v.y, 0x7632));
                const uint4 hi = make_uint4(__byte_perm(u.z, v.z, 0x5410), __byte_perm(u.z, v.z, 0x7632),
                                            __byte_perm(u.w, v.w, 0x5410), __byte_perm(u.w, v.w, 0x7632));
                uint4* dst = reinterpret_cast<uint4*>(pb) + 2 * lane;
                dst[sw] = sw ? hi : lo;
                dst[1 - sw] = sw ? lo : hi;
            }
            load(p + kPairsAhead, buf[a]);   // in flight during this pair's gather
            __syncwarp();
            const bool second = rb < rows;
#pragma unroll
            for (int k = 0; k < kSlots; ++k) {
                const int sl = lane + 32 * k;
                if (sl < S) {
                    float ta[8], tb[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        ta[j] = 0.0f;
                        tb[j] = 0.0f;
                        if (j < C) {
                            const uint16_t e = ent[k * C + j];
                            const uint32_t w = pb[e & kSrcIdxMask];
                            const float va = __uint_as_float(w << 16), vb = __uint_as_float(w & 0xFFFF0000u);
                            ta[j] = (e & kSrcNegBit) ? -va : va;
                            tb[j] = (e & kSrcNegBit) ? -vb : vb;
                        }
                    }
#pragma unroll
                    for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
                        for (int j = 0; j < w2; ++j) {
                            ta[j] += ta[j + w2];
                            tb[j] += tb[j + w2];
                        }
                    if (SS1_IN(crow0 + (size_t)ra * Kc + sl - Wc, (int64_t)gridDim.y * BN * Kc, kSiteProjWc))
                        crow0[(size_t)ra * Kc + sl] = __float2bfloat16_rn(ta[0] * scale);
                    if (second && SS1_IN(crow0 + (size_t)rb * Kc + sl - Wc, (int64_t)gridDim.y * BN * Kc, kSiteProjWc))
                        crow0[(size_t)rb * Kc + sl] = __float2bfloat16_rn(tb[0] * scale);
                }
            }
            __syncwarp();
        }
    }
}

// Any shape: one thread per output Wc[n, j], its c inputs read from global memory.
template <typename T>
__global__ void project_plain_kernel(const T* __restrict__ W, T* __restrict__ Wc, const uint16_t* __restrict__ src_tab,
                                     int64_t N, int K, int BK, int BN, int c, float scale) {
    const int S = BK / c, Kc = K / c, KC = K / BK;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N * Kc) return;
    const int64_t n = i / Kc;
    const int jj = (int)(i % Kc);
    const int kc = jj / S, s = jj % S;
    const int nb = (int)(n / BN);
    const uint16_t* e = src_tab + (((size_t)nb * KC + kc) * S + s) * c;
    float t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        t[j] = 0.0f;
        if (j < c) {
            const uint16_t ej = SS1_IN(e + j - src_tab, (N / BN) * K, kSiteProjTab) ? e[j] : (uint16_t)0;
            const int64_t wi = n * K + (int64_t)kc * BK + (ej & kSrcIdxMask);
            const float v = SS1_IN(wi, N * K, kSiteProjW) ? (float)W[wi] : 0.f;
            t[j] = (ej & kSrcNegBit) ? -v : v;
        }
    }
#pragma unroll
    for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int j = 0; j < w2; ++j) t[j] += t[j + w2];
    Wc[i] = (T)(t[0] * scale);
}

}  // namespace

bool project_fast_ok(const ss1_layer& L, const void* W, const void* Wc, int dtype) {
    (void)Wc;
    const int e = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    // the row kernel's 16-byte loads: rows and chunks start on 16-byte boundaries
    if ((L.BK * e) % 16 != 0 || (L.K * e) % 16 != 0) return false;
    return (reinterpret_cast<uintptr_t>(W) & 15u) == 0;
}

cudaError_t launch_project(const ss1_layer& L, const void* W, void* Wc, int dtype, float scale, cudaStream_t st) {
    const bool bf16 = dtype == SS1_DTYPE_BF16;
    if (!project_fast_ok(L, W, Wc, dtype)) {
        const int64_t outs = L.N * (L.K / L.c);
        const int threads = 256;
        const int64_t blocks = (outs + threads - 1) / threads;
        if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
        if (bf16)
            project_plain_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(
                (const __nv_bfloat16*)W, (__nv_bfloat16*)Wc, L.d_src, L.N, (int)L.K, L.BK, L.BN, L.c, scale);
        else
            project_plain_kernel<float><<<(unsigned)blocks, threads, 0, st>>>((const float*)W, (float*)Wc, L.d_src, L.N,
                                                                               (int)L.K, L.BK, L.BN, L.c, scale);
        return cudaGetLastError();
    }
    if (L.KC > 0x7FFFFFFF || L.NB > 65535) return cudaErrorInvalidValue;
    // split the N-block's rows only while the (N-block, K-chunk) pairs leave SMs idle
    const int64_t pairs = L.KC * L.NB, want = L.num_sms > 0 ? L.num_sms : 148;
    int splits = 1;
    while (splits * 2 <= 64 && pairs * splits < want && L.BN / (splits * 2) >= kWarps) splits *= 2;
    const int rows_per_cta = (L.BN + splits - 1) / splits;
    const dim3 grid((unsigned)L.KC, (unsigned)L.NB, (unsigned)splits);
#define SS1_PROJECT_ROWS(CC)                                                                                   \
    do {                                                                                                       \
        if (bf16)                                                                                              \
            project_pairs_kernel<CC><<<grid, kThreads, 0, st>>>((const __nv_bfloat16*)W, (__nv_bfloat16*)Wc,   \
                                                                L.d_src, (int)L.K, L.BK, L.BN, L.KC,           \
                                                                rows_per_cta, scale);                          \
        else                                                                                                   \
            project_rows_kernel<float, CC><<<grid, kThreads, 0, st>>>((const float*)W, (float*)Wc, L.d_src,    \
                                                                      (int)L.K, L.BK, L.BN, L.KC, rows_per_cta, \
                                                                      scale);                                  \
    } while (0)
    switch (L.c) {
        case 1: SS1_PROJECT_ROWS(1); break;
        case 2: SS1_PROJECT_ROWS(2); break;
        case 4: SS1_PROJECT_ROWS(4); break;
        default: SS1_PROJECT_ROWS(8); break;
    }
#undef SS1_PROJECT_ROWS
    return cudaGetLastError();
}

}  // namespace ss1

namespace ss1 {
bool handle_live(const ss1_layer* h);   // ss1_api.cu
}

extern "C" SS1_API int ss1_project(ss1_handle h, const void* W, void* Wc, int dtype, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32) return SS1_ERR_INVALID_ARG;
    if (!W || !Wc) return SS1_ERR_INVALID_ARG;
    const uintptr_t elem = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    if (((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(Wc)) & (elem - 1)) != 0) return SS1_ERR_MISALIGNED;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    // 1 / c is exact: c is a power of two
    const cudaError_t e = ss1::launch_project(*h, W, Wc, dtype, 1.0f / (float)h->c, static_cast<cudaStream_t>(stream));
    if (prev != h->device) cudaSetDevice(prev);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}
