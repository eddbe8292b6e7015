// General CUDA-core SS1 forward: sketch on chip, then an FMA GEMM against Wc.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform",
// section "Approach": the input is first sketched (signed additions reduce it by the
// compression factor c) and then multiplied with the compressed weights.
//
// This kernel runs every valid shape in bf16 or fp32 and is the fp32 path of the library.
// A CTA owns TM rows x TN columns that lie inside one N-block nb, and a range of K-chunks. Per
// K-chunk kc and per group of up to 32 slots it
//   1. sketches   Xs[m][s] = sum_j sign_j * X[m, kc*BK + k_j]   (fp32, in shared memory)
//   2. stages     Wt[s][n] = Wc[n, kc*S + s]                     (fp32, transposed)
//   3. multiplies acc[m][n] += Xs[m][s] * Wt[s][n]                (fp32 FMA, 16x16 threads)
// and finally rounds once to the output type. Sketch sums and the GEMM are both fp32, so
// for fp32 data the only roundings are those of fp32 arithmetic.
// Small batches give few output tiles, so the K-chunks are split over the CTAs of a thread-block
// cluster: each leaves its fp32 partial tile in shared memory, and after a cluster barrier CTA r
// sums rows r, r + splits, ... of all the partials in split order (the same bits every call)
// through distributed shared memory and writes Y.
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

#include <cuda_bf16.h>

namespace ss1 {
namespace {

constexpr int kThreads = 256;
constexpr int kSlotGroup = 32;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f32(float& d, float v) { d = v; }
__device__ __forceinline__ void from_f32(__nv_bfloat16& d, float v) { d = __float2bfloat16_rn(v); }

template <typename T, int TM, int TN>
__global__ void __launch_bounds__(kThreads) simt_kernel(const T* __restrict__ X, const T* __restrict__ Wc,
                                                        T* __restrict__ Y, const uint16_t* __restrict__ src,
                                                        int M, int K, int N, int c, int BK, int BN, int S, int ntiles_n) {
    constexpr int RM = TM / 16, RN = TN / 16;
    constexpr int XS_WORDS = TM * (kSlotGroup + 1), WT_WORDS = kSlotGroup * TN;
    static_assert(XS_WORDS + WT_WORDS >= TM * TN, "the partial tile fits in the staging buffers");
    __shared__ float stage_buf[XS_WORDS + WT_WORDS];
    float (*Xs)[kSlotGroup + 1] = reinterpret_cast<float (*)[kSlotGroup + 1]>(stage_buf);
    float (*Wt)[TN] = reinterpret_cast<float (*)[TN]>(stage_buf + XS_WORDS);

    const int n0 = (int)(blockIdx.x % (unsigned)ntiles_n) * TN;
    const int nb = n0 / BN;
    const int m0 = (int)(blockIdx.x / (unsigned)ntiles_n) * TM;
    const int KC = K / BK;
    const int splits = (int)gridDim.y, split = (int)blockIdx.y;
    const int kc_lo = (int)((int64_t)KC * split / splits), kc_hi = (int)((int64_t)KC * (split + 1) / splits);
    const int Kc = K / c;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;

    float acc[RM][RN];
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = 0.f;

    for (int kc = kc_lo; kc < kc_hi; ++kc) {
        const uint16_t* sblk = src + ((size_t)nb * KC + kc) * (size_t)S * c;
        for (int s0 = 0; s0 < S; s0 += kSlotGroup) {
            const int sc = min(kSlotGroup, S - s0);
            for (int i = threadIdx.x; i < TM * kSlotGroup; i += kThreads) {
                const int m = i / kSlotGroup, s = i % kSlotGroup;
                float v = 0.f;
                if (s < sc && m0 + m < M) {
                    const T* xr = X + (size_t)(m0 + m) * K + (size_t)kc * BK;
                    const uint16_t* e = sblk + (size_t)(s0 + s) * c;
                    for (int j = 0; j < c; ++j) {
                        const uint16_t t =
                            SS1_IN(e + j - src, (int64_t)(N / BN) * K, kSiteSimtTab) ? e[j] : (uint16_t)0;
                        const float x = SS1_IN(xr + (t & kSrcIdxMask) - X, (int64_t)M * K, kSiteSimtX)
                                            ? to_f32(xr[t & kSrcIdxMask])
                                            : 0.f;
                        v += (t & kSrcNegBit) ? -x : x;
                    }
                }
                Xs[m][s] = v;
            }
            for (int i = threadIdx.x; i < TN * kSlotGroup; i += kThreads) {
                const int n = i / kSlotGroup, s = i % kSlotGroup;
                const size_t wi = (size_t)(n0 + n) * Kc + (size_t)kc * S + s0 + s;
                Wt[s][n] = (s < sc && SS1_IN(wi, (int64_t)N * Kc, kSiteSimtWc)) ? to_f32(Wc[wi]) : 0.f;
            }
            __syncthreads();
            for (int s = 0; s < sc; ++s) {
                float a[RM], b[RN];
#pragma unroll
                for (int i = 0; i < RM; ++i) a[i] = Xs[ty + 16 * i][s];
#pragma unroll
                for (int j = 0; j < RN; ++j) b[j] = Wt[s][tx + 16 * j];
#pragma unroll
                for (int i = 0; i < RM; ++i)
#pragma unroll
                    for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
    if (splits == 1) {
#pragma unroll
        for (int i = 0; i < RM; ++i) {
            const int m = m0 + ty + 16 * i;
            if (m >= M) continue;
#pragma unroll
            for (int j = 0; j < RN; ++j) {
                const size_t yi = (size_t)m * N + n0 + tx + 16 * j;
                if (SS1_IN(yi, (int64_t)M * N, kSiteSimtY)) from_f32(Y[yi], acc[i][j]);
            }
        }
        return;
    }
    // the split's partial tile [TM][TN] in the staging buffers (the K loop ended on a barrier)
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) stage_buf[(ty + 16 * i) * TN + tx + 16 * j] = acc[i][j];
    ptx::cluster_sync();   // every split's partial is visible to the cluster (rank = split)
    const int rows = M - m0 < TM ? M - m0 : TM;
    for (int e = (int)ptx::cluster_ctarank() * TN + (int)threadIdx.x; e < rows * TN; e += splits * TN) {
        // element e = (row, column) of the tile; CTA r takes rows r, r + splits, ...
        if ((int)threadIdx.x >= TN) break;
        float v = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 8) {   // eight partials requested before the first is added
            float pv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                pv[q] = s0 + q < splits ? ptx::ld_cluster_f32(ptx::map_to_rank(stage_buf + e, (uint32_t)(s0 + q))) : 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (s0 + q < splits) v += pv[q];   // in split order
        }
        const size_t yi = (size_t)(m0 + e / TN) * N + n0 + e % TN;
        if (SS1_IN(yi, (int64_t)M * N, kSiteSimtY)) from_f32(Y[yi], v);
    }
    ptx::cluster_sync();   // the peers have read this CTA's partial
}

template <typename T, int TM, int TN>
cudaError_t launch_t(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    const int64_t ntn = L.N / TN, tiles = ntn * ((M + TM - 1) / TM);
    if (tiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
    // K-splits (one cluster per output tile) where the tiles alone leave most SMs idle
    int splits = 1;
    const void* fn = reinterpret_cast<const void*>(&simt_kernel<T, TM, TN>);
    ClusterFit fit;
    if (tiles < 2 * (int64_t)L.num_sms && L.KC > 1) {
        fit = cluster_fit(fn, 0, kThreads);
        splits = pick_splits(fit, (int)tiles, (int)((2 * (int64_t)L.num_sms) / tiles), L.KC);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles, (unsigned)splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = splits > 1 ? 1 : 0;
    note_launch("simt", cfg.gridDim.x, cfg.gridDim.y, splits, kThreads, 0, &fit);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, simt_kernel<T, TM, TN>, (const T*)X, (const T*)Wc, (T*)Y,
                                             (const uint16_t*)L.d_src, (int)M, (int)L.K, (int)L.N, L.c, L.BK, L.BN,
                                             L.S, (int)ntn);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T>
cudaError_t launch_dtype(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st) {
    // TN must divide BN (BN is a multiple of 16). Small M: narrow tiles for more CTAs.
    if (M <= 16) return launch_t<T, 16, 16>(L, X, Wc, Y, M, st);
    if (L.BN % 64 == 0) return launch_t<T, 64, 64>(L, X, Wc, Y, M, st);
    if (L.BN % 32 == 0) return launch_t<T, 64, 32>(L, X, Wc, Y, M, st);
    return launch_t<T, 64, 16>(L, X, Wc, Y, M, st);
}

}  // namespace

cudaError_t launch_simt(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, int dtype,
                        cudaStream_t st) {
    if (dtype == SS1_DTYPE_FP32) return launch_dtype<float>(L, X, Wc, Y, M, st);
    return launch_dtype<__nv_bfloat16>(L, X, Wc, Y, M, st);
}

}  // namespace ss1
