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
// Fast kernel: a CTA takes a tile of R rows of one N-block x one K-chunk at a time.
//   * load : W[rows, chunk] with 16-byte loads into shared memory, transposed so that one
//            32-bit word holds the same input of two rows (bf16) or of one row (fp32); the
//            word pitch is 1 mod 32, so the gathers below are free of bank conflicts.
//   * gather: lane = row pair (bf16) or row (fp32); warp w takes slots w, w + 8, ...; every
//            lane reads the slot's c sources (the same inputs for all rows of the N-block)
//            and sums them in fp32, times 1 / c, rounded once to the output type.
//   * store: the tile's outputs go through a slot-major staging buffer to 16-byte stores.
// Shapes whose rows or chunks are not 16-byte multiples take a plain kernel: one thread per
// output, reading its c inputs from global memory.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>

namespace ss1 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Word pitch of the transposed tile: >= BK and 1 mod 32.
__host__ __device__ constexpr int tile_pitch(int BK) { return ((BK + 31) / 32) * 32 + 1; }

template <bool BF16>
struct Elem;
template <>
struct Elem<true> {
    using T = __nv_bfloat16;
    static constexpr int kPerVec = 8;      // elements per 16-byte vector
    static constexpr int kRowsPerWord = 2;
};
template <>
struct Elem<false> {
    using T = float;
    static constexpr int kPerVec = 4;
    static constexpr int kRowsPerWord = 1;
};

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// Shared memory of one CTA (in 32-bit words): the transposed tile [R / rows-per-word][pitch],
// the staging buffer [S][R / rows-per-word + 1] and the chunk's slot-major table (BK entries).
template <bool BF16>
__host__ __device__ constexpr size_t smem_words(int R, int BK, int S) {
    const int units = R / Elem<BF16>::kRowsPerWord;
    return (size_t)units * tile_pitch(BK) + (size_t)S * (units + 1) + (size_t)(BK + 1) / 2;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
    project_kernel(const typename Elem<BF16>::T* __restrict__ W, typename Elem<BF16>::T* __restrict__ Wc,
                   const uint16_t* __restrict__ src_tab, int K, int BK, int BN, int c, int R, int KC,
                   int64_t units_total, float scale) {
    using E = Elem<BF16>;
    using T = typename E::T;
    constexpr int RPW = E::kRowsPerWord;
    extern __shared__ uint32_t sm[];
    const int S = BK / c;
    const int Kc = K / c;
    const int units = R / RPW;                 // row units (pairs for bf16, rows for fp32) per tile
    const int pitch = tile_pitch(BK);
    uint32_t* tile = sm;
    uint32_t* stage = tile + (size_t)units * pitch;
    const int spitch = units + 1;
    uint16_t* tab = reinterpret_cast<uint16_t*>(stage + (size_t)S * spitch);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int vecs = BK / E::kPerVec;          // 16-byte vectors per row of the chunk

    // The next unit's W tile and table entries are loaded into registers while this unit is
    // gathered and stored (at most 8 16-byte vectors per thread: 32 row pairs x 32 vectors of
    // bf16, or 32 rows x 64 vectors of fp32, over 256 threads).
    constexpr int kIters = BF16 ? 4 : 8;
    uint4 ld[8];
    uint16_t tab_next = 0;
    auto fetch = [&](int64_t u) {
        if (u >= units_total) return;
        const int kc = (int)(u % KC);
        const int64_t n0 = (u / KC) * R;
        const int nb = (int)(n0 / BN);
        if ((int)threadIdx.x < BK) tab_next = src_tab[((size_t)nb * KC + kc) * BK + threadIdx.x];
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int i = threadIdx.x + it * kThreads;
            if (i < units * vecs) {
                const int p = i % units, q = i / units;     // lanes take consecutive row units
                if (BF16) {
                    const T* r0 = W + (size_t)(n0 + 2 * p) * K + (size_t)kc * BK + q * 8;
                    ld[2 * it] = __ldg(reinterpret_cast<const uint4*>(r0));
                    ld[2 * it + 1] = __ldg(reinterpret_cast<const uint4*>(r0 + K));
                } else {
                    ld[it] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)(n0 + p) * K + (size_t)kc * BK + q * 4));
                }
            }
        }
    };
    fetch(blockIdx.x);
    for (int64_t u = blockIdx.x; u < units_total; u += gridDim.x) {
        const int64_t rt = u / KC;
        const int kc = (int)(u % KC);
        const int64_t n0 = rt * R;
        // ---- the fetched tile into shared memory, transposed; its table entries
        if ((int)threadIdx.x < BK) tab[threadIdx.x] = tab_next;
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int i = threadIdx.x + it * kThreads;
            if (i < units * vecs) {
                const int p = i % units, q = i / units;
                if (BF16) {
                    const uint4 a = ld[2 * it], b = ld[2 * it + 1];
                    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
                    uint32_t* dst = tile + (size_t)p * pitch + q * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dst[2 * e] = __byte_perm(aw[e], bw[e], 0x5410);       // inputs 2e of rows 2p, 2p+1
                        dst[2 * e + 1] = __byte_perm(aw[e], bw[e], 0x7632);   // inputs 2e+1
                    }
                } else {
                    uint32_t* dst = tile + (size_t)p * pitch + q * 4;
                    dst[0] = ld[it].x; dst[1] = ld[it].y; dst[2] = ld[it].z; dst[3] = ld[it].w;
                }
            }
        }
        __syncthreads();
        fetch(u + gridDim.x);   // in flight during the gather and the stores below
        // ---- gather: Wc[rows of unit, slot s] = (1/c) sum_j sign_j * W[rows, src_j]
        if (lane < units) {
            const uint32_t* row = tile + (size_t)lane * pitch;
            for (int s = warp; s < S; s += kWarps) {
                // the c signed terms, summed pairwise (a tree): c equal terms then add up exactly
                float lo[8], hi[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    lo[j] = 0.0f;
                    hi[j] = 0.0f;
                    if (j < c) {
                        const uint16_t e = tab[s * c + j];
                        const uint32_t w = row[e & kSrcIdxMask];
                        const bool neg = (e & kSrcNegBit) != 0;
                        const float a = BF16 ? __uint_as_float(w << 16) : __uint_as_float(w);
                        lo[j] = neg ? -a : a;
                        if (BF16) {
                            const float b = __uint_as_float(w & 0xFFFF0000u);
                            hi[j] = neg ? -b : b;
                        }
                    }
                }
#pragma unroll
                for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
                    for (int j = 0; j < w2; ++j) {
                        lo[j] += lo[j + w2];
                        hi[j] += hi[j + w2];
                    }
                stage[(size_t)s * spitch + lane] =
                    BF16 ? pack2_bf16(lo[0] * scale, hi[0] * scale) : __float_as_uint(lo[0] * scale);
            }
        }
        __syncthreads();
        // ---- store: Wc[n0 + r, kc * S + s .. + kPerVec) as 16-byte vectors; lane = row
        const int svecs = S / E::kPerVec;
        for (int i = threadIdx.x; i < R * svecs; i += kThreads) {
            const int r = i % R, sv = i / R;
            uint32_t out[4];
            if (BF16) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t w0 = stage[(size_t)(sv * 8 + 2 * e) * spitch + r / 2];
                    const uint32_t w1 = stage[(size_t)(sv * 8 + 2 * e + 1) * spitch + r / 2];
                    out[e] = (r & 1) ? __byte_perm(w0, w1, 0x7632) : __byte_perm(w0, w1, 0x5410);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) out[e] = stage[(size_t)(sv * 4 + e) * spitch + r];
            }
            *reinterpret_cast<uint4*>(Wc + (size_t)(n0 + r) * Kc + (size_t)kc * S + sv * E::kPerVec) =
                make_uint4(out[0], out[1], out[2], out[3]);
        }
        __syncthreads();
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
            const float v = (float)W[n * K + (int64_t)kc * BK + (e[j] & kSrcIdxMask)];
            t[j] = (e[j] & kSrcNegBit) ? -v : v;
        }
    }
#pragma unroll
    for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int j = 0; j < w2; ++j) t[j] += t[j + w2];
    Wc[i] = (T)(t[0] * scale);
}

int pick_rows(int BN, bool bf16) {
    const int cands_bf16[3] = {64, 32, 16}, cands_f32[2] = {32, 16};
    if (bf16) {
        for (int r : cands_bf16)
            if (BN % r == 0) return r;
    } else {
        for (int r : cands_f32)
            if (BN % r == 0) return r;
    }
    return 0;
}

}  // namespace

bool project_fast_ok(const ss1_layer& L, const void* W, const void* Wc, int dtype) {
    const int e = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    const int per_vec = 16 / e;
    if (pick_rows(L.BN, dtype == SS1_DTYPE_BF16) == 0) return false;
    if (L.BK % per_vec != 0 || L.S % per_vec != 0) return false;
    if ((L.K * e) % 16 != 0 || ((L.K / L.c) * e) % 16 != 0) return false;
    return ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(Wc)) & 15u) == 0;
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
    const int R = pick_rows(L.BN, bf16);
    const size_t smem = (bf16 ? smem_words<true>(R, L.BK, L.S) : smem_words<false>(R, L.BK, L.S)) * 4;
    const void* fn = bf16 ? reinterpret_cast<const void*>(&project_kernel<true>)
                          : reinterpret_cast<const void*>(&project_kernel<false>);
    // the largest tile (32 row units of a 256-input chunk, 256 slots at c = 1)
    constexpr int kMaxSmem = (int)(smem_words<true>(64, 256, 256) * 4);
    static_assert(smem_words<false>(32, 256, 256) * 4 <= (size_t)kMaxSmem, "fp32 tile fits the same limit");
    if (smem > (size_t)kMaxSmem) return cudaErrorInvalidValue;
    const cudaError_t ae = smem_attr_once(fn, kMaxSmem);
    if (ae != cudaSuccess) return ae;
    const int64_t units = (L.N / R) * L.KC;
    const int64_t cap = (int64_t)L.num_sms * 8;
    const int grid = (int)(units < cap ? units : cap);
    if (bf16)
        project_kernel<true><<<grid, kThreads, smem, st>>>((const __nv_bfloat16*)W, (__nv_bfloat16*)Wc, L.d_src,
                                                            (int)L.K, L.BK, L.BN, L.c, R, L.KC, units, scale);
    else
        project_kernel<false><<<grid, kThreads, smem, st>>>((const float*)W, (float*)Wc, L.d_src, (int)L.K, L.BK,
                                                             L.BN, L.c, R, L.KC, units, scale);
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
