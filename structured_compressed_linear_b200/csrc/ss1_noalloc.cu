// ss1_forward_noalloc: one SS1 layer forward whose hash tables live in a device region that the
// library reserves statically, rebuilt on the caller's stream at every call. Nothing here
// allocates memory or synchronises the device. The entry point is specified in include/ss1.h;
// the SS1 paper has no counterpart to it (it changes only where the tables are stored).
#include "ss1_internal.cuh"

#include <mutex>

namespace {

constexpr size_t kRegionBytes = (size_t)16 << 20;   // the five tables
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

constexpr size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// Bytes of the five tables of ss1_layer for `entries` = (N / BN) * K, each 256-byte aligned.
constexpr size_t region_bytes_for(size_t entries) {
    return align_up(entries * sizeof(int32_t)) + align_up(entries * sizeof(int8_t)) +
           align_up(entries * sizeof(uint16_t)) + align_up(entries * sizeof(uint2)) +
           align_up(entries * sizeof(uint16_t));
}
static_assert(region_bytes_for(SS1_NOALLOC_MAX_ENTRIES) <= kRegionBytes, "the largest accepted layer fits the region");

// One region and one status word per device context that uses this entry point.
__device__ __align__(256) uint8_t g_region[kRegionBytes];
__device__ __align__(256) int32_t g_status[64];

struct DeviceSlot {
    bool ready = false;
    uint64_t context = 0;   // id of the context the addresses below belong to
    uint8_t* region = nullptr;
    int32_t* status = nullptr;
    int num_sms = 0;
};

std::mutex g_mu;
DeviceSlot g_dev[kMaxDevices];

// One-time set-up per device context: compute capability, SM count and the regions' addresses.
// A __device__ symbol has one address per context, so the set-up runs again when the device's
// current context is not the one it ran in (after cudaDeviceReset, say).
int device_slot(int dev, DeviceSlot* out) {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceSlot& d = g_dev[dev];
    const uint64_t ctx = ss1::current_context_id();
    if (!d.ready || ctx == 0 || ctx != d.context) {
        d.ready = false;
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return SS1_ERR_CUDA;
        }
        if (major != 10) return SS1_ERR_UNSUPPORTED_DEVICE;
        void* region = nullptr;
        void* status = nullptr;
        if (cudaGetSymbolAddress(&region, g_region) != cudaSuccess ||
            cudaGetSymbolAddress(&status, g_status) != cudaSuccess || region == nullptr || status == nullptr) {
            cudaGetLastError();
            return SS1_ERR_CUDA;
        }
        d.region = static_cast<uint8_t*>(region);
        d.status = static_cast<int32_t*>(status);
        d.num_sms = sms;
        d.context = ss1::current_context_id();   // cudaGetSymbolAddress made the context current
        d.ready = true;
    }
    *out = d;
    return SS1_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" SS1_API int ss1_forward_noalloc(int64_t K, int64_t N, int c, int BK, int BN, uint64_t seed, const void* X,
                                           const void* Wc, void* Y, int64_t M, int dtype, int32_t* device_status,
                                           void* stream) {
    if (!ss1::layer_args_ok(K, N, c, BK, BN)) return SS1_ERR_INVALID_ARG;
    if (M < 0 || (dtype != SS1_DTYPE_BF16 && dtype != SS1_DTYPE_FP32)) return SS1_ERR_INVALID_ARG;
    if (M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    const int64_t entries = (N / BN) * K;
    if (entries > SS1_NOALLOC_MAX_ENTRIES) return SS1_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return SS1_OK;
    if (!X || !Wc || !Y) return SS1_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Wc, 16) || !aligned(Y, 16) || (device_status && !aligned(device_status, 4)))
        return SS1_ERR_MISALIGNED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxDevices) return SS1_ERR_UNSUPPORTED_DEVICE;
    DeviceSlot d;
    const int rc = device_slot(dev, &d);
    if (rc != SS1_OK) return rc;

    // A layer description whose tables are carved out of the region (no handle is created).
    ss1_layer L{};
    L.device = dev;
    L.num_sms = d.num_sms;
    L.K = K; L.N = N; L.c = c; L.BK = BK; L.BN = BN; L.seed = seed;
    L.S = BK / c; L.NB = (int)(N / BN); L.KC = (int)(K / BK);
    const size_t n = (size_t)entries;
    uint8_t* p = d.region;
    L.d_h = reinterpret_cast<int32_t*>(p);     p += align_up(n * sizeof(int32_t));
    L.d_g = reinterpret_cast<int8_t*>(p);      p += align_up(n * sizeof(int8_t));
    L.d_src = reinterpret_cast<uint16_t*>(p);  p += align_up(n * sizeof(uint16_t));
    L.d_gather = reinterpret_cast<uint2*>(p);  p += align_up(n * sizeof(uint2));
    L.d_slot = reinterpret_cast<uint16_t*>(p);
    L.status_host = nullptr;
    L.status_dev = device_status ? device_status : d.status;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(L.status_dev, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = ss1::launch_hashgen(L, st);
    if (e == cudaSuccess) e = ss1::launch_gather_tables(L, st);
    if (e == cudaSuccess) {
        switch (ss1::auto_kernel(L, M, dtype)) {
            case SS1_KERNEL_TC: e = ss1::launch_tc(L, X, Wc, Y, M, st); break;
            case SS1_KERNEL_SMALLM: e = ss1::launch_smallm(L, X, Wc, Y, M, st); break;
            default: e = ss1::launch_simt(L, X, Wc, Y, M, dtype, st); break;
        }
    }
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}
