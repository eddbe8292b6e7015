// ss1_test_device_timeout: the bounded-wait error path, exercised without a fault. The SS1
// pages have no counterpart; the entry point is specified in include/ss1.h. Also
// ss1_test_bounds_check, the checked build's index test on given values.
//
// One thread waits on an mbarrier that nothing arrives on, through the same bounded wait the
// forward kernels use, and writes the handle's status word the way a stalled forward kernel
// does once the limit has passed. Nothing traps; the kernel returns and the context stays usable.
#include "ss1_internal.cuh"
#include "ptx_sm100.cuh"

namespace ss1 {
bool handle_live(const ss1_layer* h);   // ss1_api.cu: a handle from ss1_create, not yet destroyed
}

namespace {

constexpr int32_t kStatusKernelSelftest = 3;   // kernel id in the status word (forward kernels use 1 and 2)
constexpr int32_t kSiteUnsatisfiedWait = 1;

__global__ void unsatisfied_wait_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    ss1::ptx::mbar_init(&bar, 1);   // one arrival would complete phase 0; none comes
    ss1::ptx::fence_mbar_init();
    if (!ss1::ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns)) {
        *(volatile int32_t*)status = (kStatusKernelSelftest << 8) | (0x80 + kSiteUnsatisfiedWait);
        __threadfence_system();
    }
}

#if SS1_CHECKED
// One thread runs the checked build's index test on (index, extent) and touches no memory
// besides the record the test writes when it fails.
__global__ void index_test_kernel(int64_t index, int64_t extent) {
    if (threadIdx.x == 0) (void)SS1_IN(index, extent, ss1::kSiteSelftest);
}
#endif

}  // namespace

extern "C" SS1_API int ss1_test_bounds_check(int64_t index, int64_t extent) {
#if SS1_CHECKED
    index_test_kernel<<<1, 32>>>(index, extent);
    return cudaGetLastError() == cudaSuccess ? SS1_OK : SS1_ERR_CUDA;
#else
    (void)index;
    (void)extent;
    return SS1_ERR_UNSUPPORTED_SHAPE;
#endif
}

extern "C" SS1_API int ss1_test_device_timeout(ss1_handle h, int64_t limit_ns, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (limit_ns < 1 || limit_ns > 2000000000) return SS1_ERR_INVALID_ARG;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    unsatisfied_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->status_dev, (uint64_t)limit_ns);
    const cudaError_t e = cudaGetLastError();
    if (prev != h->device) cudaSetDevice(prev);
    return e == cudaSuccess ? SS1_OK : SS1_ERR_CUDA;
}

extern "C" SS1_API int ss1_test_forward_timeout(ss1_handle h, const void* X, const void* Wc, void* Y, int64_t M,
                                                int64_t limit_ns, void* stream) {
    if (!ss1::handle_live(h)) return SS1_ERR_BAD_HANDLE;
    if (limit_ns < 1 || limit_ns > 2000000000 || M < 1 || M > ((int64_t)1 << 31) / 2) return SS1_ERR_INVALID_ARG;
    if (!X || !Wc || !Y) return SS1_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Wc) | reinterpret_cast<uintptr_t>(Y)) & 15u) != 0)
        return SS1_ERR_MISALIGNED;
    if (!ss1::tc3_supported(*h) || h->BK != 128 || h->c != 2 || h->NB % 2 != 0) return SS1_ERR_UNSUPPORTED_SHAPE;
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    const cudaError_t e = ss1::launch_tc3_withhold(*h, X, Wc, Y, M, (uint64_t)limit_ns, static_cast<cudaStream_t>(stream));
    if (prev != h->device) cudaSetDevice(prev);
    if (e != cudaSuccess) { cudaGetLastError(); return SS1_ERR_CUDA; }
    return SS1_OK;
}
