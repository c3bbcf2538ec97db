// Per-token top-K channel selection ("Mixture-of-Channels", sections "Dentro il
// mixture" and "Dentro MoC": per token only the K channels ranked highest by the
// SwiGLU gate stay active, as a binary mask with no threshold heuristics).
//
// One CTA per token.  The key of channel k is SiLU(z[t,k]) mapped to an
// order-preserving uint32; a 4-pass MSB-first radix select (8-bit digits,
// warp-aggregated shared-memory histograms) finds the K-th largest key, then a
// block-wide prefix sum over channel order takes the ties at that key from the
// lowest channel index up.  The keys are computed once into shared memory.
// Outputs: sel[t][k] (1 = selected) and gbuf[t][k] = SiLU(z) on selected
// channels, 0 elsewhere; optionally the
// selected channels are OR-ed into a union bitmap (bit k of word k/32).
#include "common.cuh"

namespace sffn {

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Larger float -> larger key; -0 and +0 share a key.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inverse of order_key (exact, except that -0 comes back as +0).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

constexpr int kTopkThreads = 1024;
constexpr size_t kTopkSmemKeys = 200 * 1024;   // keys staged in shared memory up to this many bytes

// SMEM: the token's keys are computed once into shared memory; otherwise every
// pass recomputes them from z (rows too long for shared memory).
template <bool SMEM>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const TopkParams p) {
    extern __shared__ uint32_t skeys[];
    __shared__ unsigned hist[256];
    __shared__ int sh[40];
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining;
    const int lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * p.d_ff;
    const float* z = p.zbuf + row;

    griddep_wait();
    griddep_launch_dependents();
    if (SMEM) {
        for (int k = threadIdx.x; k < p.d_ff; k += kTopkThreads) skeys[k] = order_key(silu_f(z[k]));
        __syncthreads();
    }
    auto key_at = [&](int k) -> uint32_t { return SMEM ? skeys[k] : order_key(silu_f(z[k])); };

    const int K = p.k;
    const bool partial = K > 0 && K < p.d_ff;
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = K;
    if (partial) {
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            if (threadIdx.x < 256) hist[threadIdx.x] = 0u;
            __syncthreads();
            for (int base = (threadIdx.x & ~31); base < p.d_ff; base += kTopkThreads) {
                const int k = base + lane;
                uint32_t digit = 0xFFFFFFFFu;
                if (k < p.d_ff) {
                    const uint32_t key = key_at(k);
                    if ((key & pmask) == prefix) digit = (key >> shift) & 0xFFu;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, digit);
                if (digit != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
            }
            __syncthreads();
            // thread i < 256 takes bin 255 - i; `before` = candidates in higher bins
            const int c = threadIdx.x < 256 ? (int)hist[255 - threadIdx.x] : 0;
            int tot = 0;
            const int before = block_exclusive_scan(c, &tot, sh);
            if (threadIdx.x < 256 && before < remaining && before + c >= remaining) {
                s_prefix = prefix | ((uint32_t)(255 - threadIdx.x) << shift);
                s_remaining = remaining - before;
            }
            __syncthreads();
            prefix = s_prefix;
            remaining = s_remaining;
            pmask |= 0xFFu << shift;
            __syncthreads();
        }
    }
    // Keys above `prefix` are all selected; `remaining` keys equal to it are
    // taken in ascending channel order.
    const int per = (p.d_ff + kTopkThreads - 1) / kTopkThreads;
    const int k0 = threadIdx.x * per, k1 = min(p.d_ff, k0 + per);
    int ties = 0;
    if (partial)
        for (int k = k0; k < k1; ++k) ties += key_at(k) == prefix;
    int tot = 0;
    int rank = block_exclusive_scan(ties, &tot, sh);
    for (int k = k0; k < k1; ++k) {
        const uint32_t key = key_at(k);
        const float gv = SMEM ? key_value(key) : silu_f(z[k]);
        bool s;
        if (!partial) {
            s = K > 0;
        } else {
            if (key == prefix) {
                s = rank < remaining;
                ++rank;
            } else {
                s = key > prefix;
            }
        }
        p.sel[row + k] = s ? 1 : 0;
        p.gbuf[row + k] = s ? gv : 0.f;
        if (s && p.ubits) atomicOr(&p.ubits[k >> 5], 1u << (k & 31));
    }
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s, bool pdl) {
    const size_t keys = (size_t)p.d_ff * sizeof(uint32_t);
    if (keys <= kTopkSmemKeys) {
        static SmemAttrCache cache;
        cudaError_t e = ensure_smem(k_topk<true>, keys, cache);
        if (e != cudaSuccess) return e;
        return launch_ex(k_topk<true>, dim3(p.n), dim3(kTopkThreads), keys, s, pdl, p);
    }
    return launch_ex(k_topk<false>, dim3(p.n), dim3(kTopkThreads), 0, s, pdl, p);
}

}  // namespace sffn
