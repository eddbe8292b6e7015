// C ABI of the SS1 layer forward: handles, argument checks, kernel choice, status words.
// The operation and every entry point are specified in include/ss1.h.
#include "ss1_internal.cuh"

#include <cuda_bf16.h>

#include <cuda.h>

#include <functional>
#include <map>
#include <mutex>
#include <new>
#include <utility>
#include <unordered_map>
#include <unordered_set>

namespace {

constexpr uint64_t kMagic = 0x5353315F4C415945ull;  // "SS1_LAYE"
constexpr int64_t kSmallMMax = 16;                   // AUTO: M <= this uses the decode path

std::mutex g_mu;
std::unordered_set<const ss1_layer*> g_live;

bool live(const ss1_layer* h) {
    std::lock_guard<std::mutex> lk(g_mu);
    return h != nullptr && g_live.count(h) != 0 && h->magic == kMagic;
}

struct PairHash {
    size_t operator()(const std::pair<const void*, uint64_t>& k) const {
        return std::hash<const void*>()(k.first) ^ (std::hash<uint64_t>()(k.second) * 0x9E3779B97F4A7C15ull);
    }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void release(ss1_layer* L) {
    if (!L) return;
    if (L->d_h) cudaFree(L->d_h);
    if (L->d_g) cudaFree(L->d_g);
    if (L->d_src) cudaFree(L->d_src);
    if (L->d_gather) cudaFree(L->d_gather);
    if (L->d_slot) cudaFree(L->d_slot);
    if (L->status_host) cudaFreeHost(L->status_host);
    L->magic = 0;
    delete L;
}

int kernel_for(const ss1_layer& L, int64_t M, int dtype) {
    if (dtype == SS1_DTYPE_FP32) return SS1_KERNEL_SIMT;
    if (M <= kSmallMMax && ss1::smallm_supported(L, M)) return SS1_KERNEL_SMALLM;
    if (ss1::tc_supported(L)) return SS1_KERNEL_TC;
    return SS1_KERNEL_SIMT;
}

template <typename T>
__global__ void bias_act_kernel(T* __restrict__ Y, const T* __restrict__ bias, int act, int64_t M, int64_t N) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= M * N) return;
    float v = (float)Y[i];
    if (bias) v += (float)bias[i % N];
    if (act == SS1_ACT_RELU) v = fmaxf(v, 0.0f);
    else if (act == SS1_ACT_GELU) v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));   // v * Phi(v)
    Y[i] = (T)v;
}

}  // namespace

namespace ss1 {

bool handle_live(const ss1_layer* h) { return live(h); }

cudaError_t launch_bias_act(void* Y, const void* bias, int act, int64_t M, int64_t N, int dtype, cudaStream_t st) {
    const int64_t n = M * N;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    if (dtype == SS1_DTYPE_BF16)
        bias_act_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(
            (__nv_bfloat16*)Y, (const __nv_bfloat16*)bias, act, M, N);
    else
        bias_act_kernel<float><<<(unsigned)blocks, threads, 0, st>>>((float*)Y, (const float*)bias, act, M, N);
    return cudaGetLastError();
}

uint64_t current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
        cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return (uint64_t)id;
}

cudaError_t smem_attr_once(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::unordered_set<std::pair<const void*, uint64_t>, PairHash> done;   // (kernel, context id)
    const uint64_t ctx = current_context_id();
    std::lock_guard<std::mutex> lk(mu);
    if (ctx != 0 && done.count({kernel, ctx})) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // the largest shared-memory carveout, so that as many CTAs as the shared memory allows are
    // resident (and the occupancy queries behind the K-split choices count them)
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    // the attribute call makes the device's context current, so its id is known from here on
    const uint64_t now = current_context_id();
    if (e == cudaSuccess && now != 0) done.insert({kernel, now});
    return e;
}

int auto_kernel(const ss1_layer& L, int64_t M, int dtype) { return kernel_for(L, M, dtype); }

ClusterFit cluster_fit(const void* fn, int smem, int threads) {
    static std::mutex mu;
    static std::map<std::pair<const void*, uint64_t>, ClusterFit> done;
    const uint64_t ctx = current_context_id();
    std::lock_guard<std::mutex> lk(mu);
    auto it = done.find({fn, ctx});
    if (ctx != 0 && it != done.end()) return it->second;
    ClusterFit f;
    cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaGetLastError();
    for (int cs = 1; cs <= 16; ++cs) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, (unsigned)cs);
        cfg.blockDim = dim3((unsigned)threads);
        cfg.dynamicSmemBytes = (size_t)smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 1;
        at[0].val.clusterDim.y = (unsigned)cs;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) == cudaSuccess) f.active[cs] = n;
        cudaGetLastError();
    }
    const uint64_t now = current_context_id();
    if (now != 0) done[{fn, now}] = f;
    return f;
}

int pick_splits(const ClusterFit& f, int groups, int want, int units) {
    int hi = want < units ? want : units;
    hi = hi > 16 ? 16 : hi;
    if (hi <= 1) return 1;
    int best = 1, best_ctas = 0;
    for (int s = hi; s >= 1; --s) {
        if (f.active[s] >= groups) return s;
        const int resident = (f.active[s] < groups ? f.active[s] : groups) * s;
        if (resident > best_ctas) { best_ctas = resident; best = s; }
    }
    return best;
}

namespace {
thread_local ss1_launch_info g_last_launch = {"", 0, 0, 0, 0, 0, {}};
}

void note_launch(const char* kernel, unsigned grid_x, unsigned grid_y, int cluster_y, int threads, int smem,
                 const ClusterFit* fit) {
    ss1_launch_info& r = g_last_launch;
    r.kernel = kernel;
    r.grid_x = (int)grid_x;
    r.grid_y = (int)grid_y;
    r.cluster_y = cluster_y;
    r.threads = threads;
    r.smem_bytes = smem;
    for (int s = 0; s <= 16; ++s) r.resident_clusters[s] = fit ? fit->active[s] : 0;
}

bool layer_args_ok(int64_t K, int64_t N, int c, int BK, int BN) {
    if (K < 1 || N < 1 || BK < 1 || BN < 1) return false;
    if (!(c == 1 || c == 2 || c == 4 || c == 8)) return false;
    if (BK > 256 || BK % c != 0 || K % BK != 0 || N % BN != 0 || BN % 16 != 0) return false;
    return K <= (int64_t)1 << 30 && N <= (int64_t)1 << 30;
}

}  // namespace ss1

#if SS1_CHECKED
namespace ss1 {
__device__ unsigned long long g_bad_access = 0;
}
#endif

extern "C" {

SS1_API int ss1_bounds_check(int* checked, uint64_t* record) {
    if (!checked || !record) return SS1_ERR_INVALID_ARG;
    *checked = SS1_CHECKED;
    *record = 0;
#if SS1_CHECKED
    unsigned long long v = 0;
    const unsigned long long zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyFromSymbol(&v, ss1::g_bad_access, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(ss1::g_bad_access, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return SS1_ERR_CUDA;
    }
    *record = v;
#endif
    return SS1_OK;
}

SS1_API int ss1_last_launch(ss1_launch_info* out) {
    if (!out) return SS1_ERR_INVALID_ARG;
    *out = ss1::g_last_launch;
    return SS1_OK;
}

SS1_API const char* ss1_strerror(int status) {
    switch (status) {
        case SS1_OK: return "ok";
        case SS1_ERR_INVALID_ARG: return "invalid argument";
        case SS1_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
        case SS1_ERR_CUDA: return "CUDA error";
        case SS1_ERR_OUT_OF_MEMORY: return "out of memory";
        case SS1_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case SS1_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait (device status set)";
        case SS1_ERR_BAD_HANDLE: return "bad or destroyed handle";
        case SS1_ERR_UNSUPPORTED_SHAPE: return "the chosen kernel does not support this shape";
        default: return "unknown status";
    }
}

SS1_API int ss1_create(int64_t K, int64_t N, int c, int BK, int BN, uint64_t seed, ss1_handle* out) {
    if (!out) return SS1_ERR_INVALID_ARG;
    *out = nullptr;
    if (K < 1 || N < 1 || BK < 1 || BN < 1) return SS1_ERR_INVALID_ARG;
    if (!(c == 1 || c == 2 || c == 4 || c == 8)) return SS1_ERR_INVALID_ARG;
    if (BK > 256 || BK % c != 0 || K % BK != 0 || N % BN != 0 || BN % 16 != 0) return SS1_ERR_INVALID_ARG;
    if (K > (int64_t)1 << 30 || N > (int64_t)1 << 30) return SS1_ERR_INVALID_ARG;
    if ((N / BN) * K >= (int64_t)1 << 31) return SS1_ERR_INVALID_ARG;   // table entries, indexed in 32 bits

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prop.major != 10) return SS1_ERR_UNSUPPORTED_DEVICE;

    ss1_layer* L = new (std::nothrow) ss1_layer{};
    if (!L) return SS1_ERR_OUT_OF_MEMORY;
    L->magic = kMagic;
    L->device = dev;
    L->num_sms = prop.multiProcessorCount;
    L->K = K; L->N = N; L->c = c; L->BK = BK; L->BN = BN; L->seed = seed;
    L->S = BK / c; L->NB = (int)(N / BN); L->KC = (int)(K / BK);

    const size_t entries = (size_t)L->NB * (size_t)K;
    if (cudaMalloc(&L->d_h, entries * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&L->d_g, entries * sizeof(int8_t)) != cudaSuccess ||
        cudaMalloc(&L->d_src, entries * sizeof(uint16_t)) != cudaSuccess ||
        cudaMalloc(&L->d_gather, entries * sizeof(uint2)) != cudaSuccess ||
        cudaMalloc(&L->d_slot, entries * sizeof(uint16_t)) != cudaSuccess ||
        cudaHostAlloc(&L->status_host, sizeof(int32_t), cudaHostAllocMapped) != cudaSuccess) {
        cudaGetLastError();
        release(L);
        return SS1_ERR_OUT_OF_MEMORY;
    }
    *L->status_host = 0;
    if (cudaHostGetDevicePointer((void**)&L->status_dev, L->status_host, 0) != cudaSuccess) {
        cudaGetLastError();
        release(L);
        return SS1_ERR_CUDA;
    }
    if (ss1::launch_hashgen(*L, 0) != cudaSuccess || ss1::launch_gather_tables(*L, 0) != cudaSuccess ||
        cudaStreamSynchronize(0) != cudaSuccess) {
        cudaGetLastError();
        release(L);
        return SS1_ERR_CUDA;
    }
    {
        std::lock_guard<std::mutex> lk(g_mu);
        g_live.insert(L);
    }
    *out = L;
    return SS1_OK;
}

SS1_API int ss1_destroy(ss1_handle h) {
    if (!h) return SS1_OK;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_live.count(h) || h->magic != kMagic) return SS1_ERR_BAD_HANDLE;
        g_live.erase(h);
    }
    const int dev = h->device;   // read before release() frees the handle
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
    cudaDeviceSynchronize();
    cudaGetLastError();
    release(h);
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
    return SS1_OK;
}

SS1_API int ss1_get_info(ss1_handle h, int64_t* K, int64_t* N, int* c, int* BK, int* BN) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    if (K) *K = h->K;
    if (N) *N = h->N;
    if (c) *c = h->c;
    if (BK) *BK = h->BK;
    if (BN) *BN = h->BN;
    return SS1_OK;
}

SS1_API int ss1_get_tables(ss1_handle h, int32_t* h_host, int8_t* g_host) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    const size_t entries = (size_t)h->NB * (size_t)h->K;
    if (h_host && cudaMemcpy(h_host, h->d_h, entries * sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return SS1_ERR_CUDA;
    }
    if (g_host && cudaMemcpy(g_host, h->d_g, entries * sizeof(int8_t), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return SS1_ERR_CUDA;
    }
    return SS1_OK;
}

SS1_API int ss1_device_status(ss1_handle h, int32_t* detail) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    const int32_t v = __atomic_exchange_n(h->status_host, 0, __ATOMIC_ACQ_REL);
    if (detail) *detail = v;
    return v == 0 ? SS1_OK : SS1_ERR_DEVICE_TIMEOUT;
}

SS1_API int ss1_select_kernel(ss1_handle h, int64_t M, int dtype, int* kernel) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    if (!kernel || M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    *kernel = kernel_for(*h, M, dtype);
    return SS1_OK;
}

SS1_API int ss1_forward_with(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M, int dtype, int kernel,
                             void* stream) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (*(volatile int32_t*)h->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
    if (M == 0) return SS1_OK;
    if (!X || !Wc || !Y) return SS1_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Wc) || !aligned16(Y)) return SS1_ERR_MISALIGNED;
    if (kernel == SS1_KERNEL_AUTO) kernel = kernel_for(*h, M, dtype);

    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    int rc = SS1_OK;
    switch (kernel) {
        case SS1_KERNEL_SIMT:
            e = ss1::launch_simt(*h, X, Wc, Y, M, dtype, st);
            break;
        case SS1_KERNEL_SMALLM:
            if (dtype != SS1_DTYPE_BF16 || !ss1::smallm_supported(*h, M)) rc = SS1_ERR_UNSUPPORTED_SHAPE;
            else e = ss1::launch_smallm(*h, X, Wc, Y, M, st);
            break;
        case SS1_KERNEL_TC:
            if (dtype != SS1_DTYPE_BF16 || !ss1::tc_supported(*h)) rc = SS1_ERR_UNSUPPORTED_SHAPE;
            else e = ss1::launch_tc(*h, X, Wc, Y, M, st);
            break;
        default:
            rc = SS1_ERR_INVALID_ARG;
    }
    if (prev != h->device) cudaSetDevice(prev);
    if (rc != SS1_OK) return rc;
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}

SS1_API int ss1_forward(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M, int dtype, void* stream) {
    return ss1_forward_with(h, X, Wc, Y, M, dtype, SS1_KERNEL_AUTO, stream);
}

SS1_API int ss1_forward_ex(ss1_handle h, const void* X, const void* Wc, const void* bias, int act, void* Y, int64_t M,
                           int dtype, int kernel, void* stream) {
    if (!live(h)) return SS1_ERR_BAD_HANDLE;
    if (act < SS1_ACT_NONE || act > SS1_ACT_GELU) return SS1_ERR_INVALID_ARG;
    if (bias && (reinterpret_cast<uintptr_t>(bias) & (dtype == SS1_DTYPE_BF16 ? 1u : 3u))) return SS1_ERR_MISALIGNED;
    if (!bias && act == SS1_ACT_NONE) return ss1_forward_with(h, X, Wc, Y, M, dtype, kernel, stream);
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (kernel == SS1_KERNEL_AUTO) kernel = kernel_for(*h, M, dtype);
    // the tensor-core kernel for c >= 2 applies bias and activation in its epilogue, before rounding
    if (kernel == SS1_KERNEL_TC && dtype == SS1_DTYPE_BF16 && ss1::tc3_supported(*h) && M > 0) {
        if (M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
        if (*(volatile int32_t*)h->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
        if (!X || !Wc || !Y) return SS1_ERR_INVALID_ARG;
        if (!aligned16(X) || !aligned16(Wc) || !aligned16(Y)) return SS1_ERR_MISALIGNED;
        int prev = -1;
        if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        const cudaError_t e = ss1::launch_tc3(*h, X, Wc, Y, M, bias, act, (cudaStream_t)stream);
        if (prev != h->device) cudaSetDevice(prev);
        if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        return SS1_OK;
    }
    // other kernels: the forward, then one elementwise pass over Y (a second rounding)
    const int rc = ss1_forward_with(h, X, Wc, Y, M, dtype, kernel, stream);
    if (rc != SS1_OK || M == 0) return rc;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    const cudaError_t e = ss1::launch_bias_act(Y, bias, act, M, h->N, dtype, (cudaStream_t)stream);
    if (prev != h->device) cudaSetDevice(prev);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}

SS1_API int ss1_chain_fused(const ss1_handle* layers, int n_layers, int* fused) {
    if (!layers || !fused || n_layers < 1 || n_layers > SS1_CHAIN_MAX_LAYERS) return SS1_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l)
        if (!live(layers[l])) return SS1_ERR_BAD_HANDLE;
    *fused = ss1::tc3_chain_ok(reinterpret_cast<const ss1_layer* const*>(layers), n_layers) ? 1 : 0;
    return SS1_OK;
}

SS1_API int ss1_chain_forward(const ss1_handle* layers, int n_layers, const void* X, const void* const* Wc,
                              const void* const* bias, const int* act, void* const* Y, int64_t M, void* stream) {
    if (!layers || !Wc || !Y || n_layers < 1 || n_layers > SS1_CHAIN_MAX_LAYERS) return SS1_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        if (!live(layers[l])) return SS1_ERR_BAD_HANDLE;
        if (l > 0 && layers[l]->K != layers[l - 1]->N) return SS1_ERR_INVALID_ARG;
        if (act && (act[l] < SS1_ACT_NONE || act[l] > SS1_ACT_GELU)) return SS1_ERR_INVALID_ARG;
        if (*(volatile int32_t*)layers[l]->status_host != 0) return SS1_ERR_DEVICE_TIMEOUT;
    }
    if (M < 0 || M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (M == 0) return SS1_OK;
    if (!X) return SS1_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        if (!Wc[l] || !Y[l]) return SS1_ERR_INVALID_ARG;
        if (!aligned16(Wc[l]) || !aligned16(Y[l]) || (bias && bias[l] && (reinterpret_cast<uintptr_t>(bias[l]) & 1u)))
            return SS1_ERR_MISALIGNED;
    }
    if (!aligned16(X)) return SS1_ERR_MISALIGNED;
    const ss1_layer* const* Ls = reinterpret_cast<const ss1_layer* const*>(layers);
    if (ss1::tc3_chain_ok(Ls, n_layers)) {   // one persistent launch for the whole chain
        int prev = -1;
        const int dev = layers[0]->device;
        if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        const cudaError_t e = ss1::launch_tc3_chain(Ls, n_layers, X, Wc, Y, bias, act, M, (cudaStream_t)stream);
        if (prev != dev) cudaSetDevice(prev);
        if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
        return SS1_OK;
    }
    // otherwise layer by layer
    for (int l = 0; l < n_layers; ++l) {
        const int rc = ss1_forward_ex(layers[l], l == 0 ? X : Y[l - 1], Wc[l], bias ? bias[l] : nullptr,
                                      act ? act[l] : SS1_ACT_NONE, Y[l], M, SS1_DTYPE_BF16, SS1_KERNEL_AUTO, stream);
        if (rc != SS1_OK) return rc;
    }
    return SS1_OK;
}

}  // extern "C"
