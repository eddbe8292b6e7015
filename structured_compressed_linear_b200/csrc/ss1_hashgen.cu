// Device generator of the SS1 hash and sign tables.
//
// "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform", section
// "Approach": K- and N-coalescing hash functions tie the weights inside one neuron's weight
// vector. The family is fixed here as: per (N-block nb, K-chunk kc) a seeded random map of
// the BK chunk inputs onto S = BK / c slots, exactly c inputs per slot, random signs.
//
// Generator (one thread per block id b = nb * KC + kc, all integer arithmetic, so the result
// is bit-reproducible on any machine):
//   key      = seed ^ mix64(b + 1)                         mix64 = SplitMix64 finaliser
//   draw(t)  = mix64(key + (t + 1) * 0x9E3779B97F4A7C15)   SplitMix64, counter form
//   shuffle  : for i = BK-1 .. 1 (draw t = BK-1-i): j = hi32(draw) * (i + 1) >> 32;
//              swap perm[i], perm[j]                       (Durstenfeld; Lemire reduction)
//   signs    : g(k) = -1 if bit 63 of draw(BK - 1 + k) is set, else +1
//   fold     : slot(k) = perm[k] mod S; the j-th source of slot s is the input k with
//              perm[k] == s + j * S
//   c == 1   : identity, all signs +1, no draws.
#include "ss1_internal.cuh"

namespace ss1 {
namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t splitmix_finalise(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void __launch_bounds__(128) hashgen_kernel(uint64_t seed, int K, int KC, int BK, int c, int S, int nblocks,
                                                      int32_t* __restrict__ h, int8_t* __restrict__ g,
                                                      uint16_t* __restrict__ src) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const int nb = b / KC, kc = b % KC;
    int32_t* hrow = h + (size_t)nb * K + (size_t)kc * BK;
    int8_t* grow = g + (size_t)nb * K + (size_t)kc * BK;
    uint16_t* sb = src + (size_t)b * S * c;

    [[maybe_unused]] const int64_t ntab = (int64_t)(nblocks / KC) * K;   // entries of each table
    if (c == 1) {
        for (int k = 0; k < BK; ++k) {
            if (!SS1_IN(hrow + k - h, ntab, kSiteHashH) || !SS1_IN(sb + k - src, ntab, kSiteHashSrc)) continue;
            hrow[k] = kc * S + k;
            grow[k] = 1;
            sb[k] = (uint16_t)k;
        }
        return;
    }

    uint8_t perm[256];   // value at each position
    uint8_t where[256];  // inverse: position -> input
    for (int k = 0; k < BK; ++k) perm[k] = (uint8_t)k;
    const uint64_t key = seed ^ splitmix_finalise((uint64_t)b + 1ull);
    uint64_t state = key;
    for (int i = BK - 1; i >= 1; --i) {
        state += kGolden;                                   // draw t = BK-1-i
        const uint64_t r = splitmix_finalise(state);
        const uint32_t j = (uint32_t)(((r >> 32) * (uint64_t)(i + 1)) >> 32);
        const uint8_t tmp = perm[i];
        perm[i] = perm[j];
        perm[j] = tmp;
    }
    for (int k = 0; k < BK; ++k) {
        state += kGolden;                                   // draw t = BK-1+k
        const uint64_t r = splitmix_finalise(state);
        const bool neg = (r >> 63) != 0;
        if (SS1_IN(hrow + k - h, ntab, kSiteHashH)) {
            hrow[k] = kc * S + (int)perm[k] % S;
            grow[k] = neg ? (int8_t)-1 : (int8_t)1;
        }
        where[perm[k]] = (uint8_t)k;
    }
    for (int s = 0; s < S; ++s) {
        for (int j = 0; j < c; ++j) {
            const int k = where[s + j * S];
            if (SS1_IN(k, BK, kSiteHashPerm) && SS1_IN(sb + s * c + j - src, ntab, kSiteHashSrc))
                sb[s * c + j] = (uint16_t)(k | (grow[k] < 0 ? kSrcNegBit : 0));
        }
    }
}

// One thread per source: the tensor-core kernel reads X[row, k] and X[row + 128, k] as one
// bf16x2 TMEM word at column k; the entry is {k, the source's sign as the bf16x2 pair (+-1, +-1)},
// ready to be added to a TMEM address and used as an FMA multiplier without further work.
__global__ void gather_table_kernel(const uint16_t* __restrict__ src, uint2* __restrict__ out, int64_t nsrc) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= nsrc) return;
    const uint16_t e = src[i];
    out[i] = make_uint2((uint32_t)(e & kSrcIdxMask), (e & kSrcNegBit) ? 0xBF80BF80u : 0x3F803F80u);
}

// One thread per (N-block, input): the input's slot inside its K-chunk and its sign, in the
// canonical input order -- what the sketch-matrix builder of the tensor-core kernel reads.
__global__ void slot_table_kernel(const int32_t* __restrict__ h, const int8_t* __restrict__ g, uint16_t* __restrict__ out,
                                  int64_t n, int K, int BK, int S) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int k = (int)(i % K);
    const int slot = h[i] - (k / BK) * S;
    if (SS1_IN(slot, S, kSiteHashSlot)) out[i] = (uint16_t)(slot | (g[i] < 0 ? kSrcNegBit : 0));
}

}  // namespace

cudaError_t launch_gather_tables(const ss1_layer& L, cudaStream_t st) {
    const int64_t nsrc = (int64_t)L.NB * L.K;
    const int threads = 256;
    const unsigned blocks = (unsigned)((nsrc + threads - 1) / threads);
    gather_table_kernel<<<blocks, threads, 0, st>>>(L.d_src, L.d_gather, nsrc);
    slot_table_kernel<<<blocks, threads, 0, st>>>(L.d_h, L.d_g, L.d_slot, nsrc, (int)L.K, L.BK, L.S);
    return cudaGetLastError();
}

cudaError_t launch_hashgen(const ss1_layer& L, cudaStream_t st) {
    const int nblocks = L.NB * L.KC;
    const int threads = 128;
    hashgen_kernel<<<(nblocks + threads - 1) / threads, threads, 0, st>>>(
        L.seed, (int)L.K, L.KC, L.BK, L.c, L.S, nblocks, L.d_h, L.d_g, L.d_src);
    return cudaGetLastError();
}

}  // namespace ss1
