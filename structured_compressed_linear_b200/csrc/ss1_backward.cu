// Backward pass of the SS1 layer: gradients of a loss with respect to X and to Wc, given dY.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Limitations": the backward pass is not made cheaper than the dense layer's. The pages give
// no formula; on the tied weight W_full[n, k] = g_nb(k) Wc[n, h_nb(k)] (nb = n / BN) matrix
// calculus gives
//
//     dX   = dY W_full                                           [M, K]
//     dWc[n, j] = sum over k with h_nb(k) == j of g_nb(k) * (dY^T X)[n, k]     [N, K / c]
//
// and both run here at the dense layer's cost, as the pages describe, on the tensor cores:
//   * input gradient : expand_t_kernel writes E = W_full^T [K, N] into the caller's workspace
//                      (each K-chunk of one N-block from a shared-memory copy of its Wc
//                      columns), then the dense tcgen05 kernel computes dX = dY E^T, both
//                      operands K-major (the reduction runs over the N neurons).
//   * weight gradient: transpose_pad_kernel writes dY^T [N, Mp] and X^T [K, Mp] (rows padded
//                      with zeros to Mp, a multiple of 64), the dense tcgen05 kernel computes
//                      G = dY^T X [N, K] (reduction over the rows), and the projection kernel
//                      sums each slot's c signed entries of G (factor 1, not 1 / c).
// fp32 data, and bf16 shapes the tensor-core kernel does not take, use a CUDA-core GEMM
// (gemm_nt_kernel) in place of the tcgen05 kernel; the accumulation is fp32 everywhere.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>

namespace ss1 {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

template <typename T>
__device__ __forceinline__ float to_f(T v) { return (float)v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v) { return (T)v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// E[kc*BK + k, n0 + r] = g_nb(k) * Wc[n0 + r, kc*S + slot_nb(k)] for one K-chunk and R neurons
// of one N-block. The R x S Wc tile is read once, coalesced, into shared memory; the E rows are
// written coalesced along n, reading the tile by column (pitch S + 1: no bank conflicts).
template <typename T>
__global__ void __launch_bounds__(256) expand_t_kernel(const T* __restrict__ Wc, T* __restrict__ E,
                                                       const int32_t* __restrict__ h, const int8_t* __restrict__ g,
                                                       int K, int N, int BK, int BN, int c, int R) {
    extern __shared__ float tile[];   // [R][S + 1]
    const int S = BK / c, Kc = K / c;
    const int kc = blockIdx.y;
    const int n0 = blockIdx.x * R;
    const int nb = n0 / BN;
    for (int i = threadIdx.x; i < R * S; i += blockDim.x) {
        const int r = i / S, s = i % S;
        const size_t wi = (size_t)(n0 + r) * Kc + (size_t)kc * S + s;
        tile[r * (S + 1) + s] = SS1_IN(wi, (int64_t)N * Kc, kSiteBwdWc) ? to_f(Wc[wi]) : 0.0f;
    }
    __syncthreads();
    const int32_t* hrow = h + (size_t)nb * K + (size_t)kc * BK;
    const int8_t* grow = g + (size_t)nb * K + (size_t)kc * BK;
    for (int i = threadIdx.x; i < BK * R; i += blockDim.x) {
        const int k = i / R, r = i % R;
        const bool tab_ok = SS1_IN(hrow + k - h, (int64_t)(N / BN) * K, kSiteBwdTab);
        const int slot = tab_ok ? hrow[k] - kc * S : 0;
        const float v = SS1_IN(slot, S, kSiteBwdSlot) ? tile[r * (S + 1) + slot] : 0.0f;
        const size_t ei = (size_t)(kc * BK + k) * N + n0 + r;
        if (SS1_IN(ei, (int64_t)K * N, kSiteBwdE)) E[ei] = from_f<T>(tab_ok && grow[k] < 0 ? -v : v);
    }
}

// out[c, r] = in[r, c] for r < rows, and 0 for rows <= r < rows_padded. in: [rows, cols].
template <typename T>
__global__ void __launch_bounds__(256) transpose_pad_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t rows,
                                                            int64_t cols, int64_t rows_padded) {
    __shared__ T t[32][33];
    const int64_t c0 = (int64_t)blockIdx.x * 32, r0 = (int64_t)blockIdx.y * 32;
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;   // 32 x 8
    for (int i = ty; i < 32; i += 8) {
        const int64_t r = r0 + i, c = c0 + tx;
        t[i][tx] = (r < rows && c < cols) ? in[r * cols + c] : from_f<T>(0.0f);
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int64_t c = c0 + i, r = r0 + tx;
        if (c < cols && r < rows_padded) out[c * rows_padded + r] = t[tx][i];
    }
}

// C[M, Nn] = A[M, Kr] B[Nn, Kr]^T on the CUDA cores, fp32 accumulation (64 x 64 tiles, 4 x 4 per thread).
template <typename T>
__global__ void __launch_bounds__(256) gemm_nt_kernel(const T* __restrict__ A, const T* __restrict__ B, T* __restrict__ C,
                                                      int64_t M, int64_t Nn, int64_t Kr) {
    __shared__ float As[16][68], Bs[16][68];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t m0 = (int64_t)blockIdx.y * 64, n0 = (int64_t)blockIdx.x * 64;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < Kr; k0 += 16) {
        for (int i = threadIdx.x; i < 64 * 16; i += 256) {
            const int r = i / 16, kk = i % 16;
            const int64_t k = k0 + kk;
            As[kk][r] = (m0 + r < M && k < Kr) ? to_f(A[(m0 + r) * Kr + k]) : 0.0f;
            Bs[kk][r] = (n0 + r < Nn && k < Kr) ? to_f(B[(n0 + r) * Kr + k]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
            if (m < M && n < Nn) C[m * Nn + n] = from_f<T>(acc[i][j]);
        }
}

int pick_rows(int BN) { return BN % 64 == 0 ? 64 : (BN % 32 == 0 ? 32 : 16); }

int64_t padded_rows(int64_t M) { return (M + 63) / 64 * 64; }

// The dense tcgen05 kernel (c = 1 layer kernel) as a plain GEMM C[rows, Nout] = A[rows, Kr] B[Nout, Kr]^T
// (bf16, both K-major): a layer description with the identity hash over Kr inputs and Nout outputs.
bool dense_tc_ok(int64_t rows, int64_t Nout, int64_t Kr) {
    return Nout % 128 == 0 && Kr % 64 == 0 && rows >= 1 && (rows + 127) / 128 <= 65535 && Kr <= (1 << 30) &&
           Nout <= (1 << 30);
}

cudaError_t dense_tc(const ss1_layer& L, const void* A, const void* B, void* C, int64_t rows, int64_t Nout, int64_t Kr,
                     cudaStream_t st) {
    ss1_layer P{};
    P.device = L.device;
    P.num_sms = L.num_sms;
    P.K = Kr;
    P.N = Nout;
    P.c = 1;
    P.BK = Kr % 256 == 0 ? 256 : (Kr % 128 == 0 ? 128 : 64);
    P.BN = 128;
    P.S = P.BK;
    P.NB = (int)(Nout / 128);
    P.KC = (int)(Kr / P.BK);
    P.status_dev = L.status_dev;
    return launch_tc(P, A, B, C, rows, st);
}

template <typename T>
cudaError_t gemm_simt(const void* A, const void* B, void* C, int64_t M, int64_t Nn, int64_t Kr, cudaStream_t st) {
    const int64_t gx = (Nn + 63) / 64, gy = (M + 63) / 64;
    if (gx > 0x7FFFFFFF || gy > 65535) return cudaErrorInvalidValue;
    gemm_nt_kernel<T><<<dim3((unsigned)gx, (unsigned)gy), 256, 0, st>>>((const T*)A, (const T*)B, (T*)C, M, Nn, Kr);
    return cudaGetLastError();
}

template <typename T>
cudaError_t expand_t(const ss1_layer& L, const void* Wc, void* E, cudaStream_t st) {
    const int R = pick_rows(L.BN);
    const size_t smem = (size_t)R * (L.S + 1) * sizeof(float);
    const void* fn = reinterpret_cast<const void*>(&expand_t_kernel<T>);
    // the largest tile: 64 neurons x (256 + 1) slots (c = 1, BK = 256)
    const cudaError_t ae = smem_attr_once(fn, 64 * 257 * (int)sizeof(float));
    if (ae != cudaSuccess) return ae;
    expand_t_kernel<T><<<dim3((unsigned)(L.N / R), (unsigned)L.KC), 256, smem, st>>>(
        (const T*)Wc, (T*)E, L.d_h, L.d_g, (int)L.K, (int)L.N, L.BK, L.BN, L.c, R);
    return cudaGetLastError();
}

template <typename T>
cudaError_t transpose_pad(const void* in, void* out, int64_t rows, int64_t cols, int64_t rows_padded, cudaStream_t st) {
    const int64_t gx = (cols + 31) / 32, gy = (rows_padded + 31) / 32;
    if (gx > 0x7FFFFFFF || gy > 65535) return cudaErrorInvalidValue;
    transpose_pad_kernel<T><<<dim3((unsigned)gx, (unsigned)gy), 256, 0, st>>>((const T*)in, (T*)out, rows, cols,
                                                                             rows_padded);
    return cudaGetLastError();
}

}  // namespace

size_t backward_input_workspace(const ss1_layer& L, int dtype) {
    const size_t e = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    return align_up((size_t)L.K * (size_t)L.N * e);
}

size_t backward_weight_workspace(const ss1_layer& L, int64_t M, int dtype) {
    const size_t e = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    const size_t Mp = (size_t)padded_rows(M);
    return align_up((size_t)L.N * Mp * e) + align_up((size_t)L.K * Mp * e) + align_up((size_t)L.N * (size_t)L.K * e);
}

cudaError_t launch_backward_input(const ss1_layer& L, const void* dY, const void* Wc, void* dX, int64_t M, int dtype,
                                  void* ws, cudaStream_t st) {
    const bool bf16 = dtype == SS1_DTYPE_BF16;
    cudaError_t e = bf16 ? expand_t<__nv_bfloat16>(L, Wc, ws, st) : expand_t<float>(L, Wc, ws, st);
    if (e != cudaSuccess) return e;
    // dX[M, K] = dY[M, N] E[K, N]^T
    if (bf16 && dense_tc_ok(M, L.K, L.N)) return dense_tc(L, dY, ws, dX, M, L.K, L.N, st);
    return bf16 ? gemm_simt<__nv_bfloat16>(dY, ws, dX, M, L.K, L.N, st) : gemm_simt<float>(dY, ws, dX, M, L.K, L.N, st);
}

cudaError_t launch_backward_weight(const ss1_layer& L, const void* X, const void* dY, void* dWc, int64_t M, int dtype,
                                   void* ws, cudaStream_t st) {
    const bool bf16 = dtype == SS1_DTYPE_BF16;
    const size_t e = bf16 ? 2 : 4;
    const int64_t Mp = padded_rows(M);
    uint8_t* p = static_cast<uint8_t*>(ws);
    void* dYt = p;                                                  // [N, Mp]
    void* Xt = p + align_up((size_t)L.N * Mp * e);                   // [K, Mp]
    void* G = static_cast<uint8_t*>(Xt) + align_up((size_t)L.K * Mp * e);   // [N, K] = dY^T X
    cudaError_t err = bf16 ? transpose_pad<__nv_bfloat16>(dY, dYt, M, L.N, Mp, st)
                           : transpose_pad<float>(dY, dYt, M, L.N, Mp, st);
    if (err == cudaSuccess)
        err = bf16 ? transpose_pad<__nv_bfloat16>(X, Xt, M, L.K, Mp, st) : transpose_pad<float>(X, Xt, M, L.K, Mp, st);
    if (err != cudaSuccess) return err;
    // G[N, K] = dY^T[N, Mp] (X^T[K, Mp])^T
    if (bf16 && dense_tc_ok(L.N, L.K, Mp))
        err = dense_tc(L, dYt, Xt, G, L.N, L.K, Mp, st);
    else
        err = bf16 ? gemm_simt<__nv_bfloat16>(dYt, Xt, G, L.N, L.K, Mp, st) : gemm_simt<float>(dYt, Xt, G, L.N, L.K, Mp, st);
    if (err != cudaSuccess) return err;
    // dWc[n, j] = sum over the slot's inputs k of g(k) G[n, k]
    return launch_project(L, G, dWc, dtype, 1.0f, st);
}

}  // namespace ss1

namespace ss1 {
bool handle_live(const ss1_layer* h);   // ss1_api.cu
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Makes h's device current for the call and restores the caller's afterwards.
struct DeviceScope {
    int prev = -1;
    bool ok = true;
    explicit DeviceScope(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) { cudaGetLastError(); ok = false; }
    }
    void restore(int dev) {
        if (ok && prev >= 0 && prev != dev) cudaSetDevice(prev);
    }
};

}  // namespace

extern "C" SS1_API int ss1_backward_workspace(ss1_handle h, int64_t M, int dtype, size_t* input_bytes,
                                              size_t* weight_bytes) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (input_bytes) *input_bytes = ss1::backward_input_workspace(*h, dtype);
    if (weight_bytes) *weight_bytes = ss1::backward_weight_workspace(*h, M, dtype);
    return SS1_OK;
}

extern "C" SS1_API int ss1_backward_input(ss1_handle h, const void* dY, const void* Wc, void* dX, int64_t M, int dtype,
                                          void* workspace, size_t workspace_bytes, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (*(volatile int32_t*)h->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
    if (M == 0) return SS1_OK;
    if (!dY || !Wc || !dX || !workspace) return SS1_ERR_INVALID_ARG;
    if (workspace_bytes < ss1::backward_input_workspace(*h, dtype)) return SS1_ERR_INVALID_ARG;
    if (!aligned16(dY) || !aligned16(Wc) || !aligned16(dX) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return SS1_ERR_MISALIGNED;
    DeviceScope ds(h->device);
    if (!ds.ok) return SS1_ERR_CUDA;
    const cudaError_t e =
        ss1::launch_backward_input(*h, dY, Wc, dX, M, dtype, workspace, static_cast<cudaStream_t>(stream));
    ds.restore(h->device);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}

extern "C" SS1_API int ss1_backward_weight(ss1_handle h, const void* X, const void* dY, void* dWc, int64_t M, int dtype,
                                           void* workspace, size_t workspace_bytes, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (*(volatile int32_t*)h->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
    if (!dWc || (M > 0 && (!X || !dY || !workspace))) return SS1_ERR_INVALID_ARG;
    if (!aligned16(dWc)) return SS1_ERR_MISALIGNED;
    DeviceScope ds(h->device);
    if (!ds.ok) return SS1_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    const size_t e_bytes = dtype == SS1_DTYPE_BF16 ? 2 : 4;
    if (M == 0) {   // no rows: the gradient is zero
        e = cudaMemsetAsync(dWc, 0, (size_t)h->N * (size_t)(h->K / h->c) * e_bytes, static_cast<cudaStream_t>(stream));
    } else {
        if (workspace_bytes < ss1::backward_weight_workspace(*h, M, dtype)) { ds.restore(h->device); return SS1_ERR_INVALID_ARG; }
        if (!aligned16(X) || !aligned16(dY) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
            ds.restore(h->device);
            return SS1_ERR_MISALIGNED;
        }
        e = ss1::launch_backward_weight(*h, X, dY, dWc, M, dtype, workspace, static_cast<cudaStream_t>(stream));
    }
    ds.restore(h->device);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}
