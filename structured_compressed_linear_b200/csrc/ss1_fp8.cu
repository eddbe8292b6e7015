// FP8 (E4M3) compressed weights with one float scale per output neuron.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform": section
// "Limitations" lists quantised SS1 kernels as not built, and section "Measured effects" reports
// post-training quantisation of SS1 models. The pages fix no format; this library stores
//
//     Wc_deq[n, j] = scale[n] * e4m3(Wq[n, j])      (OCP E4M3: bias 7, 3 mantissa bits, max 448)
//
// and computes the layer on Wc_deq. Decode-sized batches are bound by reading Wc, so one byte
// per weight halves that bound. ss1_forward_fp8 runs the tensor-core decode kernel with the
// E4M3 stages widened to bf16 on chip (exact) and the scale applied to each neuron's fp32 sum.
// ss1_quantize_fp8 makes (Wq, scale) from bf16 or fp32 weights: scale[n] = max_j |Wc[n, j]| / 448
// (1 for a zero row) and Wq = E4M3(Wc / scale), round to nearest even, saturating at 448.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace ss1 {
bool handle_live(const ss1_layer* h);   // ss1_api.cu
}

namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float as_f(T v) { return (float)v; }
template <>
__device__ __forceinline__ float as_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// One CTA per row: the row's largest magnitude (a block reduction), its scale, then the codes.
template <typename T>
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const T* __restrict__ Wc, uint8_t* __restrict__ Wq,
                                                                 float* __restrict__ scale, int64_t Kc) {
    __shared__ float red[kThreads / 32];
    const T* row = Wc + (size_t)blockIdx.x * Kc;
    uint8_t* out = Wq + (size_t)blockIdx.x * Kc;
    float m = 0.0f;
    for (int64_t j = threadIdx.x; j < Kc; j += kThreads) m = fmaxf(m, fabsf(as_f(row[j])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = m;
    __syncthreads();
    float amax = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;   // correctly rounded, as IEEE division
    if (threadIdx.x == 0) scale[blockIdx.x] = sc;
    for (int64_t j = threadIdx.x; j < Kc; j += kThreads) {
        const float q = __fdiv_rn(as_f(row[j]), sc);
        out[j] = (uint8_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);   // round to nearest even
    }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" SS1_API int ss1_forward_fp8(ss1_handle h, const void* X, const void* Wq, const float* scale, void* Y,
                                       int64_t M, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (M < 0 || M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (*(volatile int32_t*)h->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
    if (M == 0) return SS1_OK;
    if (!X || !Wq || !scale || !Y) return SS1_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(scale, 4)) return SS1_ERR_MISALIGNED;
    if (!ss1::dec_fp8_supported(*h, M)) return SS1_ERR_UNSUPPORTED_SHAPE;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    const cudaError_t e = ss1::launch_dec_fp8(*h, X, Wq, scale, Y, M, static_cast<cudaStream_t>(stream));
    if (prev != h->device) cudaSetDevice(prev);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}

extern "C" SS1_API int ss1_quantize_fp8(const void* Wc, int dtype, int64_t N, int64_t Kc, void* Wq, float* scale,
                                        void* stream) {
    if (N < 0 || Kc < 1 || N > 0x7FFFFFFF || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32))
        return SS1_ERR_INVALID_ARG;
    if (N == 0) return SS1_OK;
    if (!Wc || !Wq || !scale) return SS1_ERR_INVALID_ARG;
    if (!aligned(Wc, dtype == SS1_DTYPE_BF16 ? 2 : 4) || !aligned(scale, 4)) return SS1_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == SS1_DTYPE_BF16)
        quantize_rows_kernel<__nv_bfloat16><<<(unsigned)N, kThreads, 0, st>>>((const __nv_bfloat16*)Wc, (uint8_t*)Wq,
                                                                           scale, Kc);
    else
        quantize_rows_kernel<float><<<(unsigned)N, kThreads, 0, st>>>((const float*)Wc, (uint8_t*)Wq, scale, Kc);
    if (cudaGetLastError() != cudaSuccess) return SS1_ERR_CUDA;
    return SS1_OK;
}
