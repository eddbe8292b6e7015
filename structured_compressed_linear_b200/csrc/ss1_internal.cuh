// Internal declarations shared by the SS1 CUDA sources (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ss1.h"

// Kernel-side table entry: the chunk-local input index of one slot source and its sign.
//   bits 0..7  : k_local in [0, BK)  (BK <= 256)
//   bit  15    : 1 if the sign is -1
// Layout of the slot-major table: src[((nb * KC + kc) * S + s) * c + j], j = 0..c-1, where
// the j-th source of slot s is the input whose permuted position is s + j * S.
static constexpr uint16_t kSrcNegBit = 0x8000u;
static constexpr uint16_t kSrcIdxMask = 0x00FFu;

// Checked build. Compiled with SS1_CHECKED=1 (the debug library libss1_checked.so, which stands
// in for a memory checker), every global-memory access that a kernel addresses by its own index
// arithmetic first tests the element index against the extent of the buffer, in elements of
// that buffer. A failed test records (site << 48) | index in one device word (the first failure
// only; ss1_bounds_check reads and clears it) and the access is skipped: a load yields 0, a store
// or copy is not made, and a wait on a skipped copy ends at its time limit. Tile copies by TMA
// are bounded by their tensor maps in hardware and are not tested. In the normal build a test is
// the constant true and compiles away.
#ifndef SS1_CHECKED
#define SS1_CHECKED 0
#endif

namespace ss1 {
enum CheckSite : int {
    kSiteSimtTab = 1, kSiteSimtX, kSiteSimtWc, kSiteSimtY,
    kSiteSmallmTab, kSiteSmallmX, kSiteSmallmWc, kSiteSmallmY,
    kSiteDecTab, kSiteDecX, kSiteDecY, kSiteDecScale,
    kSiteProjTab, kSiteProjW, kSiteProjWc,
    kSiteTc3Tab, kSiteTc3Bias, kSiteTc2Tab, kSiteTc2Wc, kSiteTc2Y,
    kSiteBwdWc, kSiteBwdTab, kSiteBwdSlot, kSiteBwdE,
    kSiteHashH, kSiteHashPerm, kSiteHashSrc, kSiteHashSlot,
    kSiteSelftest = 63,
};
#if SS1_CHECKED
extern __device__ unsigned long long g_bad_access;
__device__ __forceinline__ bool check_span(int64_t i, int64_t len, int64_t n, int site) {
    if (i >= 0 && len >= 0 && i + len <= n) return true;
    atomicCAS(&g_bad_access, 0ull, ((unsigned long long)site << 48) | ((unsigned long long)i & 0xFFFFFFFFFFFFull));
    return false;
}
#endif
}  // namespace ss1

#if SS1_CHECKED
#define SS1_IN(i, n, site) (::ss1::check_span((int64_t)(i), 1, (int64_t)(n), (site)))
#define SS1_SPAN_IN(i, len, n, site) (::ss1::check_span((int64_t)(i), (int64_t)(len), (int64_t)(n), (site)))
#else
#define SS1_IN(i, n, site) true
#define SS1_SPAN_IN(i, len, n, site) true
#endif

struct ss1_layer {
    uint64_t magic;
    int device;
    int num_sms;
    int64_t K, N;
    int c, BK, BN, S, NB, KC;
    uint64_t seed;
    int32_t* d_h;        // [NB][K] compressed column of input k in block nb
    int8_t* d_g;         // [NB][K] sign of input k in block nb
    uint16_t* d_src;     // [NB][KC][S][c] slot-major sources (see above)
    uint2* d_gather;     // [NB][KC][BK] per source (slot-major): {k, bf16x2 multiplier (+-1, +-1)}
    uint16_t* d_slot;    // [NB][K] per input: slot inside its chunk (bits 0..7) | kSrcNegBit if the sign is -1
    int32_t* status_host;  // pinned, host-mapped status word (0 = ok)
    int32_t* status_dev;   // device alias of status_host
};

namespace ss1 {

// Device status codes written by kernels with bounded waits: (kernel id << 8) | wait site.
enum : int32_t { kStatusKernelTC = 1, kStatusKernelDec = 2 };

// The kernel ss1_forward picks for (M, dtype) (SS1_KERNEL_TC, _SIMT or _SMALLM).
int auto_kernel(const ss1_layer& L, int64_t M, int dtype);
// The shape checks of ss1_create.
bool layer_args_ok(int64_t K, int64_t N, int c, int BK, int BN);

// Unique id of the CUDA context current on this thread (cuCtxGetId), 0 if none is current yet.
// Ids are never reused, so a context created after a device reset gets a new one.
uint64_t current_context_id();

// How many clusters of cs CTAs (cluster dimensions (1, cs, 1)) the device keeps resident at once
// for a kernel, cs = 1 .. 16 (16 is a non-portable size; 0 where a size does not fit at all).
// Clusters are placed whole inside one GPC, so this is not the CTA slots divided by cs. Looked
// up once per (kernel, context).
struct ClusterFit {
    int active[17] = {};
};
ClusterFit cluster_fit(const void* fn, int smem, int threads);
// K-splits per output group when each group's splits form one cluster: the largest count up to
// `want` (and `units`, at most 16) whose `groups` clusters all fit on the device at once; where
// none does, the one that keeps the most CTAs resident.
int pick_splits(const ClusterFit& f, int groups, int want, int units);

// Records the shape of a layer kernel's launch for ss1_last_launch (per host thread). `fit` is the
// occupancy query behind a K-split choice, or null.
void note_launch(const char* kernel, unsigned grid_x, unsigned grid_y, int cluster_y, int threads, int smem,
                 const ClusterFit* fit);

// Y[m, n] = act(Y[m, n] + bias[n]) in place (bias may be null), for kernels without the fused epilogue.
cudaError_t launch_bias_act(void* Y, const void* bias, int act, int64_t M, int64_t N, int dtype, cudaStream_t st);

// Raises `kernel`'s dynamic shared-memory limit to `bytes` and asks for the largest shared-memory
// carveout, in the current context. The attributes belong to a context, so they are set once per
// (kernel, context); later calls return at once.
cudaError_t smem_attr_once(const void* kernel, int bytes);

cudaError_t launch_hashgen(const ss1_layer& L, cudaStream_t st);
// Derives d_gather from d_src (run after launch_hashgen).
cudaError_t launch_gather_tables(const ss1_layer& L, cudaStream_t st);

// General CUDA-core path: any valid shape, bf16 or fp32.
cudaError_t launch_simt(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, int dtype,
                        cudaStream_t st);

// Decode-sized M (bf16): streams Wc once. The tensor-core decode kernel takes N-blocks of 128;
// the CUDA-core one the rest.
bool dec_supported(const ss1_layer& L, int64_t M);
// The same kernel with FP8 (E4M3) Wc and one float scale per neuron (Y = scale[n] * sum).
bool dec_fp8_supported(const ss1_layer& L, int64_t M);
cudaError_t launch_dec_fp8(const ss1_layer& L, const void* X, const void* Wq, const float* scale, void* Y, int64_t M,
                           cudaStream_t st);
cudaError_t launch_dec(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st);
bool smallm_supported(const ss1_layer& L, int64_t M);
cudaError_t launch_smallm(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M,
                          cudaStream_t st);

// Tensor-core path (bf16, tcgen05 + TMEM + TMA).
bool tc_supported(const ss1_layer& L);
// Transposed-tile variant (c >= 2): 128 neurons x 256 rows per tile, sketch gathered from TMEM.
bool tc2_supported(const ss1_layer& L);
cudaError_t launch_tc2(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st);
// Sketch-as-GEMM variant (c >= 2): the sketch of each chunk is a tcgen05.mma with an on-chip
// 0/+-1 matrix; 128 rows x one or two N-blocks per tile.
bool tc3_supported(const ss1_layer& L);
// bias: bf16 [N] or null; act: 0 none, 1 ReLU, 2 GELU (applied to the fp32 sum before rounding).
cudaError_t launch_tc3(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, const void* bias, int act,
                       cudaStream_t st);
// Test of the time-out path: the same launch with every wait limited to wait_ns, and CTA 0's
// first build warp withholding its arrival for the third sketch segment, so a wait runs out.
cudaError_t launch_tc3_withhold(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M,
                                uint64_t wait_ns, cudaStream_t st);
// A chain of up to four layers in one persistent launch (layer l + 1 reads layer l's Y): every
// layer tc3-supported with the first layer's BK, c and N-block grouping, K of l + 1 == N of l.
bool tc3_chain_ok(const ss1_layer* const* Ls, int n);
cudaError_t launch_tc3_chain(const ss1_layer* const* Ls, int n, const void* X, const void* const* Wc, void* const* Y,
                             const void* const* bias, const int* act, int64_t M, cudaStream_t st);
cudaError_t launch_tc(const ss1_layer& L, const void* X, const void* Wc, void* Y, int64_t M, cudaStream_t st);

// Dense -> SS1 projection (bf16 or fp32): Wc[n, j] = scale * sum_{k : h(k) = j} g(k) W[n, k]
// (scale = 1 / c for the projection, 1 for the weight gradient's tied sum).
bool project_fast_ok(const ss1_layer& L, const void* W, const void* Wc, int dtype);
cudaError_t launch_project(const ss1_layer& L, const void* W, void* Wc, int dtype, float scale, cudaStream_t st);

}  // namespace ss1
