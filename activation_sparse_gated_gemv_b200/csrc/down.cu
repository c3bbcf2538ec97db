// Gathered down projection with a deterministic two-phase reduction:
//   y[t,:] = sum over listed channels k of h[k][t] * W_down[k,:]
// ("Mixture-of-Channels", section "Scomporre i risultati": at inference only
// the K active channels are multiplied and accumulated, so only their W_down
// rows are read.)
//
// Grid = (column slices of 512 outputs) x (chunks of the active list).  Every
// CTA rebuilds the list's prefix over the gate CTAs' segments, takes an equal
// share of the M listed channels, streams the 512-column piece of each of its
// rows (16-byte L1-bypassing loads, four rows in flight per thread) and writes
// an fp32 partial.  The last CTA to finish a column slice (ticket counter)
// adds the partials in chunk order and stores y.  The chunk count shrinks on
// the device with M, so a short list does not pay for many partials; the
// result depends only on M, never on timing.
#include "common.cuh"

namespace sffn {

constexpr int kSliceCols = 512;

struct DownSmem {
    size_t prefix, rows, red, total;
};
__host__ __device__ inline DownSmem down_smem_layout(int nt, int g1, int max_rows, int rg) {
    DownSmem L;
    size_t o = 0;
    L.prefix = o; o += (((size_t)g1 + 1) * sizeof(int) + 15) & ~(size_t)15;
    L.rows = o;   o += ((size_t)max_rows * sizeof(int) + 15) & ~(size_t)15;
    L.red = o;    o += (size_t)rg * nt * kSliceCols * sizeof(float);
    L.total = o;
    return L;
}

template <class T, int NT>
__global__ void __launch_bounds__(kThreads) k_down(const DownParams p) {
    constexpr int V = Elem<T>::kVec;
    constexpr int TPR = kSliceCols / V;      // threads per row
    constexpr int RG = kThreads / TPR;       // row groups
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int sh[40];
    __shared__ int s_last;
    const DownSmem L = down_smem_layout(NT, p.g1, p.max_rows, RG);
    int* prefix = reinterpret_cast<int*>(smem + L.prefix);
    int* rows_k = reinterpret_cast<int*>(smem + L.rows);
    float* red = reinterpret_cast<float*>(smem + L.red);

    griddep_wait();
    griddep_launch_dependents();

    int carry = 0;
    for (int b0 = 0; b0 < p.g1; b0 += kThreads) {
        const int b = b0 + threadIdx.x;
        const int c = b < p.g1 ? p.seg_count[b] : 0;
        int tot = 0;
        const int ex = block_exclusive_scan(c, &tot, sh);
        if (b < p.g1) prefix[b] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) prefix[p.g1] = carry;
    const int M = carry;
    const int chunks_eff = max(1, min(p.chunks, (M + p.min_rows - 1) / p.min_rows));
    if ((int)blockIdx.y >= chunks_eff) return;
    const int q0 = (int)((long long)M * blockIdx.y / chunks_eff);
    const int q1 = (int)((long long)M * (blockIdx.y + 1) / chunks_eff);
    int rows = q1 - q0;
    // rows <= max(min_rows, ceil(d_ff / chunks)) by construction; guard anyway
    // (record it and contribute nothing, so the ticket protocol still completes).
    if (rows > p.max_rows) {
        if (threadIdx.x == 0) atomicOr(p.status, (int)kStatusDownRows);
        rows = 0;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < rows; i += kThreads) {
        const int q = q0 + i;
        int lo = 0, hi = p.g1;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= q) lo = mid; else hi = mid;
        }
        rows_k[i] = p.lst_idx[lo * p.cpb + (q - prefix[lo])];
    }
    __syncthreads();

    const T* wdn = static_cast<const T*>(p.wdn);
    const int rg = threadIdx.x / TPR, tc = threadIdx.x - rg * TPR;
    const int col = blockIdx.x * kSliceCols + tc * V;
    const bool colok = col < p.d;
    for (int t0 = 0; t0 < p.n; t0 += NT) {
        const int nt = min(NT, p.n - t0);
        float acc[NT][V];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < V; ++e) acc[t][e] = 0.f;
        int i = rg;
        for (; i + 3 * RG < rows; i += 4 * RG) {
            int kk[4];
            uint4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) kk[u] = rows_k[i + u * RG];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                w[u] = colok ? ld_stream(wdn + (size_t)kk[u] * p.d + col) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float wf[V];
                unpack<T>(w[u], wf);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float hv = t < nt ? p.lst_h[(size_t)kk[u] * p.n + t0 + t] : 0.f;
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[t][e] = fmaf(hv, wf[e], acc[t][e]);
                }
            }
        }
        for (; i < rows; i += RG) {
            const int k = rows_k[i];
            const uint4 w = colok ? ld_stream(wdn + (size_t)k * p.d + col) : make_uint4(0u, 0u, 0u, 0u);
            float wf[V];
            unpack<T>(w, wf);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float hv = t < nt ? p.lst_h[(size_t)k * p.n + t0 + t] : 0.f;
#pragma unroll
                for (int e = 0; e < V; ++e) acc[t][e] = fmaf(hv, wf[e], acc[t][e]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < V; ++e) red[((size_t)rg * NT + t) * kSliceCols + tc * V + e] = acc[t][e];
        __syncthreads();
        for (int idx = threadIdx.x; idx < NT * kSliceCols; idx += kThreads) {
            const int t = idx / kSliceCols, c = idx - t * kSliceCols;
            const int gc = blockIdx.x * kSliceCols + c;
            if (t < nt && gc < p.d) {
                float s = 0.f;
#pragma unroll
                for (int g = 0; g < RG; ++g) s += red[((size_t)g * NT + t) * kSliceCols + c];
                p.part[((size_t)blockIdx.y * p.n + t0 + t) * p.d + gc] = s;
            }
        }
    }

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.tickets[blockIdx.x], 1u) == (unsigned)chunks_eff - 1u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    T* y = static_cast<T*>(p.y);
    for (int idx = threadIdx.x; idx < p.n * kSliceCols; idx += kThreads) {
        const int t = idx / kSliceCols;
        const int gc = blockIdx.x * kSliceCols + (idx - t * kSliceCols);
        if (gc < p.d) {
            float s = 0.f;
            for (int ch = 0; ch < chunks_eff; ++ch) s += __ldcg(&p.part[((size_t)ch * p.n + t) * p.d + gc]);
            y[(size_t)t * p.d + gc] = from_f32<T>(s);
        }
    }
    if (threadIdx.x == 0) p.tickets[blockIdx.x] = 0u;
}

int down_slice_cols(int /*wdtype*/) { return kSliceCols; }

int down_max_rows(int d_ff, int chunks, int min_rows) {
    const int c = chunks > 0 ? chunks : 1;
    const int per = (d_ff + c - 1) / c;
    return per > min_rows ? per : min_rows;
}

size_t down_smem_bytes(int wdtype, int nt, int g1, int max_rows) {
    const int V = wdtype == 0 ? 8 : 4;
    const int rg = kThreads / (kSliceCols / V);
    return down_smem_layout(nt, g1, max_rows, rg).total;
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
    if (p.max_rows < down_max_rows(p.d_ff, p.chunks, p.min_rows) ||
        smem < down_smem_bytes(wdtype, nt, p.g1, p.max_rows))
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
