// Per-token top-K channel selection ("Mixture-of-Channels", sections "Dentro il
// mixture" and "Dentro MoC": per token only the K channels ranked highest by the
// SwiGLU gate stay active, as a binary mask with no threshold heuristics), and
// per-token top-p selection ("PrunePath", abstract: a softmax-normalised
// routing distribution with a cumulative-mass threshold).
//
// One CTA per token.  The key of channel k is SiLU(z[t,k]) mapped to an
// order-preserving uint32; a 4-pass MSB-first radix select (8-bit digits,
// per-warp shared-memory histograms) finds the K-th largest key, then a
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
constexpr size_t kTopkSmemKeys = 180 * 1024;   // keys staged in shared memory up to this many bytes

// Fixed-point scale 2^S of the top-p masses: a token's total stays below 2^31.
__host__ __device__ inline int topp_scale_bits(int d_ff) {
    int s = 0;
    while (s < 24 && ((long long)d_ff << (s + 1)) < (1ll << 31)) ++s;
    return s;
}

// SMEM: the token's keys are computed once into shared memory; otherwise every
// pass recomputes them from z (rows too long for shared memory).
// Top-K (p.mode 0): key = order of SiLU(z); each channel counts 1; keep K.
// Top-p (p.mode 1): key = order of z; each channel weighs
//   m_k = round(exp(z_k - max z) 2^S) (integer, so sums are exact and the
//   choice reproducible); keep the shortest prefix by descending key whose
//   mass reaches ceil(p sum_k m_k).
template <bool SMEM>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const TopkParams p) {
    extern __shared__ uint32_t dyn[];
    unsigned* whist = dyn;                                // [32 warps][256 bins]
    uint32_t* skeys = dyn + 32 * 256;                     // [d_ff] (SMEM)
    __shared__ unsigned hist[256];
    __shared__ int sh[40];
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining;
    __shared__ unsigned s_binw;                           // weight of the final pass's chosen bin
    __shared__ unsigned s_red[33];
    const int lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * p.d_ff;
    const float* z = p.zbuf + row;
    const bool topp = p.mode == 1;

    griddep_wait();
    griddep_launch_dependents();
    auto make_key = [&](int k) -> uint32_t { return order_key(topp ? z[k] : silu_f(z[k])); };
    if (SMEM) {
        // eight loads of z in flight per thread before the keys are made
        constexpr int U = 8;
        for (int k0 = threadIdx.x; k0 < p.d_ff; k0 += U * kTopkThreads) {
            float zv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = k0 + u * kTopkThreads;
                zv[u] = k < p.d_ff ? __ldcg(z + k) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = k0 + u * kTopkThreads;
                if (k < p.d_ff) skeys[k] = order_key(topp ? zv[u] : silu_f(zv[u]));
            }
        }
        __syncthreads();
    }
    auto key_at = [&](int k) -> uint32_t { return SMEM ? skeys[k] : make_key(k); };

    // top-p: the largest gate value, the masses and their total
    float zmax = 0.f, scale = 0.f;
    if (topp) {
        uint32_t mk = 0u;
        for (int k = threadIdx.x; k < p.d_ff; k += kTopkThreads) mk = max(mk, key_at(k));
#pragma unroll
        for (int o = 16; o; o >>= 1) mk = max(mk, __shfl_xor_sync(0xffffffffu, mk, o));
        if (lane == 0) s_red[threadIdx.x >> 5] = mk;
        __syncthreads();
        if (threadIdx.x < 32) {
            uint32_t v = s_red[threadIdx.x];
#pragma unroll
            for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (threadIdx.x == 0) s_red[32] = v;
        }
        __syncthreads();
        zmax = key_value(s_red[32]);
        scale = (float)(1 << topp_scale_bits(p.d_ff));
        __syncthreads();
    }
    auto mass_of = [&](uint32_t key) -> unsigned { return __float2uint_rn(expf(key_value(key) - zmax) * scale); };

    int target = p.k;                                     // top-K: channels; top-p: mass
    if (topp) {
        unsigned tm = 0u;
        for (int k = threadIdx.x; k < p.d_ff; k += kTopkThreads) tm += mass_of(key_at(k));
#pragma unroll
        for (int o = 16; o; o >>= 1) tm += __shfl_xor_sync(0xffffffffu, tm, o);
        if (lane == 0) s_red[threadIdx.x >> 5] = tm;
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned v = s_red[threadIdx.x];
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (threadIdx.x == 0) s_red[32] = v;
        }
        __syncthreads();
        const unsigned total = s_red[32];
        target = (int)min((double)total, ceil((double)p.p * (double)total));
        __syncthreads();
    }
    const bool partial = topp ? target > 0 : (target > 0 && target < p.d_ff);
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = target;
    if (partial) {
        unsigned* mine = whist + (threadIdx.x >> 5) * 256;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = threadIdx.x; i < 32 * 256; i += kTopkThreads) whist[i] = 0u;
            __syncthreads();
            // per-warp histograms (integer weights: the sums are exact in any order)
            for (int k = threadIdx.x; k < p.d_ff; k += kTopkThreads) {
                const uint32_t key = key_at(k);
                if ((key & pmask) == prefix) atomicAdd(&mine[(key >> shift) & 0xFFu], topp ? mass_of(key) : 1u);
            }
            __syncthreads();
            if (threadIdx.x < 256) {
                unsigned h = 0u;
#pragma unroll 8
                for (int w = 0; w < 32; ++w) h += whist[w * 256 + threadIdx.x];
                hist[threadIdx.x] = h;
            }
            __syncthreads();
            // thread i < 256 takes bin 255 - i; `before` = weight in higher bins
            const int c = threadIdx.x < 256 ? (int)hist[255 - threadIdx.x] : 0;
            int tot = 0;
            const int before = block_exclusive_scan(c, &tot, sh);
            if (threadIdx.x < 256 && c > 0 && before < remaining && before + c >= remaining) {
                s_prefix = prefix | ((uint32_t)(255 - threadIdx.x) << shift);
                s_remaining = remaining - before;
                s_binw = (unsigned)c;
            }
            __syncthreads();
            prefix = s_prefix;
            remaining = s_remaining;
            pmask |= 0xFFu << shift;
            __syncthreads();
        }
    }
    // Keys above `prefix` are all selected; of the keys equal to it, taken in
    // ascending channel order: `remaining` (top-K) or enough to cover the
    // remaining mass (top-p: equal keys weigh the same).
    int take = remaining;
    if (topp && partial) {
        const unsigned m_tie = mass_of(prefix);
        take = m_tie ? (int)((remaining + m_tie - 1) / m_tie) : 0;
    }
    // Channels tied at the boundary key: when all of them are kept (the usual
    // case) the choice needs no ranks and the writes stream in channel order.
    // The last pass's chosen bin holds exactly the keys equal to the boundary,
    // so its weight gives their number (top-p: every tie weighs m_tie).
    int nties = 0;
    if (partial) {
        const unsigned m_tie = topp ? mass_of(prefix) : 1u;
        if (m_tie) {
            nties = (int)(s_binw / m_tie);
        } else {
            int c = 0;
            for (int k = threadIdx.x; k < p.d_ff; k += kTopkThreads) c += key_at(k) == prefix;
            int tot0 = 0;
            block_exclusive_scan(c, &tot0, sh);
            nties = tot0;
        }
    }
    if (!partial || nties <= take) {
        // a warp covers 32 consecutive channels, one word of the union bitmap
        const int warp = threadIdx.x >> 5;
        for (int base = warp * 32; base < p.d_ff; base += kTopkThreads) {
            const int k = base + lane;
            bool s = false;
            if (k < p.d_ff) {
                const uint32_t key = key_at(k);
                const float gv = topp ? silu_f(key_value(key)) : (SMEM ? key_value(key) : silu_f(z[k]));
                s = partial ? key >= prefix : (!topp && target > 0);
                p.sel[row + k] = s ? 1 : 0;
                p.gbuf[row + k] = s ? gv : 0.f;
            }
            const unsigned m = __ballot_sync(0xffffffffu, s);
            if (lane == 0 && m && p.ubits) atomicOr(&p.ubits[base >> 5], m);
        }
        return;
    }
    const int per = (p.d_ff + kTopkThreads - 1) / kTopkThreads;
    const int k0 = threadIdx.x * per, k1 = min(p.d_ff, k0 + per);
    int ties = 0;
    for (int k = k0; k < k1; ++k) ties += key_at(k) == prefix;
    int tot = 0;
    int rank = block_exclusive_scan(ties, &tot, sh);
    for (int k = k0; k < k1; ++k) {
        const uint32_t key = key_at(k);
        const float gv = topp ? silu_f(key_value(key)) : (SMEM ? key_value(key) : silu_f(z[k]));
        bool s;
        if (!partial) {
            s = !topp && target > 0;
        } else {
            if (key == prefix) {
                s = rank < take;
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
    const size_t whist = 32 * 256 * sizeof(unsigned);
    const size_t keys = (size_t)p.d_ff * sizeof(uint32_t);
    if (keys <= kTopkSmemKeys) {
        static SmemAttrCache cache;
        cudaError_t e = ensure_smem(k_topk<true>, whist + keys, cache);
        if (e != cudaSuccess) return e;
        return launch_ex(k_topk<true>, dim3(p.n), dim3(kTopkThreads), whist + keys, s, pdl, p);
    }
    static SmemAttrCache cache2;
    cudaError_t e = ensure_smem(k_topk<false>, whist, cache2);
    if (e != cudaSuccess) return e;
    return launch_ex(k_topk<false>, dim3(p.n), dim3(kTopkThreads), whist, s, pdl, p);
}

}  // namespace sffn
