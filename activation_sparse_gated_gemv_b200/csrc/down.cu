// Gathered down projection with a deterministic two-phase reduction:
//   y[t,:] = sum over listed channels k of h[k][t] * W_down[k,:]
// ("Mixture-of-Channels", section "Scomporre i risultati": at inference only
// the K active channels are multiplied and accumulated, so only their W_down
// rows are read.)
//
// Grid = (column slices of 512 outputs) x (chunks).  Chunk c takes the list
// segments of gate CTAs [c*g1/CH, (c+1)*g1/CH): their counts and (speculatively)
// their whole slot ranges of channel ids are read in one round trip, then
// compacted in shared memory.  Each thread reads a 16-byte piece of the
// 512-column slice of its row group's listed W_down rows, up to 16 rows in
// flight per thread (L1-bypassing loads), multiplies by h and accumulates in
// fp32; row groups are added in a fixed order and the CTA's partial goes to
// global memory.  The last CTA of each column slice
// (ticket counter) adds the chunk partials in chunk order and stores y, so y is
// bitwise reproducible.
#include "common.cuh"

namespace sffn {

constexpr int kSliceCols = 512;

struct DownSmem {
    size_t cnt, idx, rowk, red, total;
};
__host__ __device__ inline DownSmem down_smem_layout(int nt, int nseg, int cpb, int rg) {
    DownSmem L;
    size_t o = 0;
    const size_t cap = (size_t)nseg * cpb;
    L.cnt = o;   o += (((size_t)nseg + 1) * 2 * sizeof(int) + 15) & ~(size_t)15;   // counts, prefix
    L.idx = o;   o += (cap * sizeof(int) + 15) & ~(size_t)15;
    L.rowk = o;  o += (cap * sizeof(int) + 15) & ~(size_t)15;
    L.red = o;   o += (size_t)rg * nt * kSliceCols * sizeof(float);
    L.total = o;
    return L;
}

template <class T, int NT>
__global__ void __launch_bounds__(kThreads, 2) k_down(const DownParams p) {
    constexpr int V = Elem<T>::kVec;
    constexpr int TPR = kSliceCols / V;             // threads per row
    constexpr int RG = kThreads / TPR;              // row groups
    constexpr int UB = NT == 1 ? 16 : NT == 2 ? 8 : 4;   // rows in flight per thread
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_last;
    const int nseg_max = (p.g1 + p.chunks - 1) / p.chunks;
    const DownSmem L = down_smem_layout(NT, nseg_max, p.cpb, RG);
    int* cnt = reinterpret_cast<int*>(smem + L.cnt);
    int* pre = cnt + nseg_max + 1;
    int* idx = reinterpret_cast<int*>(smem + L.idx);
    int* rowk = reinterpret_cast<int*>(smem + L.rowk);
    float* red = reinterpret_cast<float*>(smem + L.red);

    const int seg0 = (int)((long long)blockIdx.y * p.g1 / p.chunks);
    const int seg1 = (int)((long long)(blockIdx.y + 1) * p.g1 / p.chunks);
    const int nseg = seg1 - seg0;
    const int col0 = blockIdx.x * kSliceCols;
    const int ncols = min(kSliceCols, p.d - col0);
    const T* wdn = static_cast<const T*>(p.wdn);

    griddep_wait();
    griddep_launch_dependents();

    // Counts and the segments' whole slot ranges, in one round trip.  Counts
    // and channel ids come from the gate kernel: a count beyond its segment's
    // slots, or a channel outside its segment's range, raises kStatusBounds
    // and is dropped (clamped, or its row skipped) instead of being followed.
    for (int i = threadIdx.x; i < nseg; i += kThreads) {
        const int c = p.seg_count[seg0 + i];
        const int room = max(0, min(p.cpb, p.d_ff - (seg0 + i) * p.cpb));
        if (c < 0 || c > room) raise_status(p.status, p.hstatus, kStatusBounds);
        cnt[i] = min(max(c, 0), room);
    }
    for (int i = threadIdx.x; i < nseg * p.cpb; i += kThreads) {
        const int slot = seg0 * p.cpb + i;
        idx[i] = slot < p.d_ff ? p.lst_idx[slot] : 0;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        int carry = 0;
        for (int b0 = 0; b0 < nseg; b0 += 32) {
            const int b = b0 + threadIdx.x;
            const int c = b < nseg ? cnt[b] : 0;
            int x = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if ((int)threadIdx.x >= o) x += y;
            }
            if (b < nseg) pre[b] = carry + x - c;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (threadIdx.x == 0) pre[nseg] = carry;
    }
    __syncthreads();
    const int rows = pre[nseg];
    for (int i = threadIdx.x; i < nseg * p.cpb; i += kThreads) {
        const int j = i / p.cpb, o = i - j * p.cpb;
        if (o < cnt[j]) {
            const int k = idx[i], lo = (seg0 + j) * p.cpb;
            const bool ok = k >= lo && k < lo + p.cpb && k < p.d_ff;
            if (!ok) raise_status(p.status, p.hstatus, kStatusBounds);
            rowk[pre[j] + o] = ok ? k : -1;
        }
    }
    __syncthreads();

    const int rg = threadIdx.x / TPR, tc = threadIdx.x - rg * TPR;
    const bool colok = tc * V < ncols;
    const T* wcol = wdn + col0 + tc * V;
    for (int t0 = 0; t0 < p.n; t0 += NT) {
        const int nt = min(NT, p.n - t0);
        float2 acc[NT][V / 2];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < V / 2; ++e) acc[t][e] = make_float2(0.f, 0.f);
        for (int i0 = rg; i0 < rows; i0 += UB * RG) {
            uint4 w[UB];
            float h[UB][NT];
#pragma unroll
            for (int u = 0; u < UB; ++u) {
                const int i = i0 + u * RG;
                const int k = i < rows ? rowk[i] : -1;        // -1: no row, or one a check dropped
                const bool in = k >= 0;
                w[u] = (in && colok) ? ld_stream(wcol + (size_t)k * p.d) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int t = 0; t < NT; ++t) h[u][t] = (in && t < nt) ? p.lst_h[(size_t)k * p.n + t0 + t] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < UB; ++u) {
                float wf[V];
                unpack<T>(w[u], wf);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float2 hh = make_float2(h[u][t], h[u][t]);
#pragma unroll
                    for (int e = 0; e < V / 2; ++e)
                        acc[t][e] = __ffma2_rn(make_float2(wf[2 * e], wf[2 * e + 1]), hh, acc[t][e]);
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < V / 2; ++e)
                *reinterpret_cast<float2*>(red + ((size_t)rg * NT + t) * kSliceCols + tc * V + 2 * e) = acc[t][e];
        __syncthreads();
        for (int i = threadIdx.x; i < NT * (kSliceCols / 4); i += kThreads) {
            const int t = i / (kSliceCols / 4), c = (i - t * (kSliceCols / 4)) * 4;
            if (t < nt && c < ncols) {
                float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    const float4 v = *reinterpret_cast<const float4*>(red + ((size_t)r * NT + t) * kSliceCols + c);
                    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
                }
                *reinterpret_cast<float4*>(p.part + ((size_t)blockIdx.y * p.n + t0 + t) * p.d + col0 + c) = s;
            }
        }
    }

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.tickets[blockIdx.x], 1u) == (unsigned)p.chunks - 1u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // Sum the chunk partials in chunk order.  Item = (token, 4 columns); when
    // there are fewer items than threads, G thread groups take interleaved
    // chunks and their sums are added in group order.
    T* y = static_cast<T*>(p.y);
    constexpr int C4 = kSliceCols / 4;
    const int items = p.n * C4;
    const int G = items >= kThreads ? 1 : kThreads / items;
    const int per_round = kThreads / G;
    float4* gsum = reinterpret_cast<float4*>(red);                // [G][per_round]
    const size_t stride = (size_t)p.n * p.d / 4;
    for (int base = 0; base < items; base += per_round) {
        const int item = base + (int)threadIdx.x % per_round;
        const int grp = (int)threadIdx.x / per_round;
        const int t = item / C4, c = (item - t * C4) * 4;
        const bool ok = item < items && c < ncols && grp < G;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ok) {
            const float4* src = reinterpret_cast<const float4*>(p.part + (size_t)t * p.d + col0 + c);
            // 16 loads in flight per batch; the last batch is predicated, so a
            // short chunk list still costs a single round trip.
            for (int ch = grp; ch < p.chunks; ch += 16 * G) {
                float4 v[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int c2 = ch + q * G;
                    v[q] = c2 < p.chunks ? __ldcg(src + (size_t)c2 * stride) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    if (ch + q * G < p.chunks) {
                        s.x += v[q].x; s.y += v[q].y; s.z += v[q].z; s.w += v[q].w;
                    }
                }
            }
        }
        if (G > 1) {
            __syncthreads();
            if (grp < G) gsum[grp * per_round + (int)threadIdx.x % per_round] = s;
            __syncthreads();
            if (grp == 0 && ok) {
                for (int q = 1; q < G; ++q) {
                    const float4 v = gsum[q * per_round + (int)threadIdx.x % per_round];
                    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
                }
            }
        }
        if (grp == 0 && ok) {
            T* dst = y + (size_t)t * p.d + col0 + c;
            dst[0] = from_f32<T>(s.x);
            dst[1] = from_f32<T>(s.y);
            dst[2] = from_f32<T>(s.z);
            dst[3] = from_f32<T>(s.w);
        }
    }
    if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;
}

int down_slice_cols(int /*wdtype*/) { return kSliceCols; }

size_t down_smem_bytes(int wdtype, int nt, int nseg, int cpb) {
    const int V = wdtype == 0 ? 8 : 4;
    const int rg = kThreads / (kSliceCols / V);
    return down_smem_layout(nt, nseg, cpb, rg).total;
}

template <class T, int NT>
static cudaError_t launch_down_t(const DownParams& p, int slices, size_t smem, cudaStream_t s, bool pdl) {
    auto kern = k_down<T, NT>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(slices, p.chunks), dim3(kThreads), smem, s, pdl, p);
}

cudaError_t launch_down(int wdtype, const DownParams& p, int nt, int slices, size_t smem, cudaStream_t s,
                        bool pdl) {
    const int nseg = (p.g1 + p.chunks - 1) / p.chunks;
    if (p.chunks < 1 || p.chunks > p.g1 || smem < down_smem_bytes(wdtype, nt, nseg, p.cpb))
        return cudaErrorInvalidValue;
    if (wdtype == 0) {
        switch (nt) {
            case 1: return launch_down_t<bf16, 1>(p, slices, smem, s, pdl);
            case 2: return launch_down_t<bf16, 2>(p, slices, smem, s, pdl);
            case 4: return launch_down_t<bf16, 4>(p, slices, smem, s, pdl);
            default: return launch_down_t<bf16, 8>(p, slices, smem, s, pdl);
        }
    }
    switch (nt) {
        case 1: return launch_down_t<float, 1>(p, slices, smem, s, pdl);
        case 2: return launch_down_t<float, 2>(p, slices, smem, s, pdl);
        case 4: return launch_down_t<float, 4>(p, slices, smem, s, pdl);
        default: return launch_down_t<float, 8>(p, slices, smem, s, pdl);
    }
}

}  // namespace sffn
