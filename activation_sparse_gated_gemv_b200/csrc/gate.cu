// Gate-first kernels.
//
// k_gate: one pass over a CTA's contiguous channel range [c0, c0 + cpb):
//   1. gate   z[t,k] = <x_t, W_gate[:,k]> (dense row of d) or <u_t, B[:,k]> (LoPA row of r),
//             or the top-K kernel's decision read back (preselected);
//   2. select active iff z > tau (threshold) -- "Model Casting and Low-Parameter
//             Gating" (abstract): the gate is evaluated first and only channels
//             whose activation is non-zero go on;
//   3. up     for a channel active in any token, h[k][t] = g[t,k] <x_t, W_up[:,k]>
//             (0 for tokens that did not select k) -- the only W_up rows read are
//             the active ones ("Mixture-of-Channels", section "Dentro il mixture");
//   4. list   ordered compaction of the CTA's active channels into its own fixed
//             slot range of the list (block-wide prefix sum), so the list is in
//             ascending channel order with no global atomics.
// One warp owns RW channel rows at a time; each lane streams 16-byte chunks with
// L1-bypassing loads and the warp reduces with shuffles.  x (and LoPA's u) sit
// in shared memory as fp32 for the token tile.
//
// k_lopa_u: LoPA's first stage u = x A ("Model Casting and Low-Parameter
// Gating", abstract: a low-FLOPs parameterization of the gating matrix, read as
// the rank-r product A B).  A split-d grid writes partial sums; the last CTA of
// each column group (ticket counter) adds them in split order, so u is
// deterministic.
#include "common.cuh"

namespace sffn {

// acc[r][t] = <row r, xs[t]> for r < nr; every lane ends with the full sums.
// Rows are w0 + r * wstride (elements), cpr 16-byte chunks each; xs is fp32
// [NT][xstride] in shared memory.
template <class WT, int NT, int RW>
__device__ __forceinline__ void warp_dot(const WT* __restrict__ w0, size_t wstride, int nr, int cpr,
                                         const float* xs, int xstride, float (&acc)[RW][NT]) {
    constexpr int V = Elem<WT>::kVec;
    constexpr int UB = RW >= 16 ? 1 : 16 / RW;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][t] = 0.f;
    for (int cb = lane; cb < cpr; cb += 32 * UB) {
        uint4 wv[UB][RW];
#pragma unroll
        for (int u = 0; u < UB; ++u)
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int c = cb + 32 * u;
                wv[u][r] = (c < cpr && r < nr) ? ld_stream(w0 + (size_t)r * wstride + (size_t)c * V)
                                               : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            const int c = cb + 32 * u;
            if (c < cpr) {
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    float wf[V];
                    unpack<WT>(wv[u][r], wf);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float4* xp = reinterpret_cast<const float4*>(xs + t * xstride + c * V);
                        float a = acc[r][t];
#pragma unroll
                        for (int q = 0; q < V / 4; ++q) {
                            const float4 xv = xp[q];
                            a = fmaf(wf[4 * q + 0], xv.x, a);
                            a = fmaf(wf[4 * q + 1], xv.y, a);
                            a = fmaf(wf[4 * q + 2], xv.z, a);
                            a = fmaf(wf[4 * q + 3], xv.w, a);
                        }
                        acc[r][t] = a;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[r][t] = warp_sum(acc[r][t]);
}

// Shared-memory carve-up of k_gate (host and device agree through this).
struct GateSmem {
    size_t xs, us, mask, flag, scan, total;
};
__host__ __device__ inline GateSmem gate_smem_layout(int nt, int d, int r, int gate_kind, int cpb,
                                                     int mw) {
    GateSmem L;
    size_t o = 0;
    L.xs = o;   o += (size_t)nt * d * sizeof(float);
    L.us = o;   o += gate_kind == kGateLopa ? (size_t)nt * r * sizeof(float) : 0;
    L.mask = o; o += (size_t)cpb * mw * sizeof(uint32_t);
    L.flag = o; o += ((size_t)cpb + 15) & ~(size_t)15;
    L.scan = o; o += 40 * sizeof(int);
    L.total = o;
    return L;
}

template <class T, int NT, int RW, int GATE>
__global__ void __launch_bounds__(kThreads, 2) k_gate(const GateParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int V = Elem<T>::kVec;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * p.cpb;
    const int nslots = max(0, min(p.cpb, p.d_ff - c0));
    const GateSmem L = gate_smem_layout(NT, p.d, p.r, GATE, p.cpb, p.mw);
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    float* us = reinterpret_cast<float*>(smem + L.us);
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + L.mask);
    uint8_t* flag = reinterpret_cast<uint8_t*>(smem + L.flag);
    int* scan_sh = reinterpret_cast<int*>(smem + L.scan);

    const T* x = static_cast<const T*>(p.x);
    const T* wg = static_cast<const T*>(p.wg);
    const T* bcm = static_cast<const T*>(p.bcm);
    const T* wup = static_cast<const T*>(p.wup);
    const int cpr_d = p.d / V;
    const int cpr_r = p.r / V;
    const int ntiles = (p.n + NT - 1) / NT;

    griddep_wait();
    griddep_launch_dependents();

    for (int i = threadIdx.x; i < p.cpb; i += kThreads) flag[i] = 0;
    for (int i = threadIdx.x; i < p.cpb * p.mw; i += kThreads) smask[i] = 0u;

    for (int tile = 0; tile < ntiles; ++tile) {
        const int t0 = tile * NT;
        const int nt = min(NT, p.n - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < NT * cpr_d; i += kThreads) {
            const int t = i / cpr_d, c = i - t * cpr_d;
            float f[V];
            if (t < nt) {
                unpack<T>(*reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * p.d + (size_t)c * V), f);
            } else {
#pragma unroll
                for (int q = 0; q < V; ++q) f[q] = 0.f;
            }
            float4* dst = reinterpret_cast<float4*>(xs + (size_t)t * p.d + (size_t)c * V);
#pragma unroll
            for (int q = 0; q < V / 4; ++q)
                dst[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
        }
        if (GATE == kGateLopa) {
            for (int i = threadIdx.x; i < NT * p.r; i += kThreads) {
                const int t = i / p.r, c = i - t * p.r;
                us[i] = t < nt ? p.u[(size_t)(t0 + t) * p.r + c] : 0.f;
            }
        }
        __syncthreads();

        for (int s0 = warp * RW; s0 < nslots; s0 += kWarps * RW) {
            const int nr = min(RW, nslots - s0);
            float z[RW][NT];
            if (GATE == kGateDense) {
                warp_dot<T, NT, RW>(wg + (size_t)(c0 + s0) * p.d, (size_t)p.d, nr, cpr_d, xs, p.d, z);
            } else if (GATE == kGateLopa) {
                warp_dot<T, NT, RW>(bcm + (size_t)(c0 + s0) * p.r, (size_t)p.r, nr, cpr_r, us, p.r, z);
            } else {
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int t = 0; t < NT; ++t) z[r][t] = 0.f;
            }
#pragma unroll
            for (int rr = 0; rr < RW; ++rr) {
                if (rr < nr) {
                    const int s = s0 + rr, k = c0 + s;
                    if (p.out == kOutWriteZ) {
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            if (lane == t && t < nt) p.zbuf[(size_t)(t0 + t) * p.d_ff + k] = z[rr][t];
                    } else {
                        uint32_t tokmask = 0u;
                        float gv[NT];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            bool a = false;
                            gv[t] = 0.f;
                            if (t < nt) {
                                if (GATE == kGatePreselected) {
                                    const size_t o = (size_t)(t0 + t) * p.d_ff + k;
                                    a = p.sel[o] != 0;
                                    gv[t] = p.gbuf[o];
                                } else {
                                    a = z[rr][t] > p.tau;
                                    gv[t] = z[rr][t] - p.tau;
                                }
                            }
                            tokmask |= (a ? 1u : 0u) << t;
                        }
                        if (tokmask != 0u || p.force_all) {
                            float uu[1][NT];
                            warp_dot<T, NT, 1>(wup + (size_t)k * p.d, (size_t)p.d, 1, cpr_d, xs, p.d, uu);
#pragma unroll
                            for (int t = 0; t < NT; ++t)
                                if (lane == t && t < nt)
                                    p.lst_h[(size_t)k * p.n + t0 + t] =
                                        ((tokmask >> t) & 1u) ? gv[t] * uu[0][t] : 0.f;
                            if (lane == 0) {
                                flag[s] = 1;
                                smask[s * p.mw + (t0 >> 5)] |= tokmask << (t0 & 31);
                            }
                        } else if (ntiles > 1) {
#pragma unroll
                            for (int t = 0; t < NT; ++t)
                                if (lane == t && t < nt) p.lst_h[(size_t)k * p.n + t0 + t] = 0.f;
                        }
                    }
                }
            }
        }
    }
    if (p.out == kOutWriteZ) return;

    // Ordered compaction: thread i owns slots [i*per, (i+1)*per).
    __syncthreads();
    const int per = (nslots + kThreads - 1) / kThreads;
    const int sb = threadIdx.x * per;
    int cnt = 0;
    for (int i = 0; i < per; ++i)
        if (sb + i < nslots && flag[sb + i]) ++cnt;
    int total = 0;
    int pos = block_exclusive_scan(cnt, &total, scan_sh);
    for (int i = 0; i < per; ++i) {
        const int s = sb + i;
        if (s < nslots && flag[s]) {
            p.lst_idx[c0 + pos] = c0 + s;
            for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + s) * p.mw + w] = smask[s * p.mw + w];
            ++pos;
        }
    }
    if (threadIdx.x == 0) p.seg_count[blockIdx.x] = total;
}

// ---------------------------------------------------------------------------
// LoPA stage 1: u = x A.  grid = (d splits, r column groups).

template <class T, int NT>
__global__ void __launch_bounds__(kThreads) k_lopa_u(const LopaUParams p) {
    constexpr int V = Elem<T>::kVec;
    extern __shared__ __align__(16) unsigned char smem[];
    float* red = reinterpret_cast<float*>(smem);   // [RG][NT][cols]
    __shared__ int s_last;
    const T* x = static_cast<const T*>(p.x);
    const T* a = static_cast<const T*>(p.a);
    const int tpr = p.cols_per_cta / V;            // threads per row
    const int rg_n = kThreads / tpr;               // row groups
    const int rg = threadIdx.x / tpr, tc = threadIdx.x - rg * tpr;
    const int j0 = blockIdx.x * p.rows_per_cta;
    const int j1 = min(p.d, j0 + p.rows_per_cta);
    const int col = blockIdx.y * p.cols_per_cta + tc * V;
    const bool active = rg < rg_n && col < p.r;
    const int ncols = min(p.cols_per_cta, p.r - blockIdx.y * p.cols_per_cta);

    griddep_wait();
    griddep_launch_dependents();

    for (int t0 = 0; t0 < p.n; t0 += NT) {
        const int nt = min(NT, p.n - t0);
        float acc[NT][V];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < V; ++e) acc[t][e] = 0.f;
        if (active) {
            for (int j = j0 + rg; j < j1; j += rg_n) {
                float wf[V];
                unpack<T>(ld_stream(a + (size_t)j * p.r + col), wf);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float xv = t < nt ? to_f32<T>(x[(size_t)(t0 + t) * p.d + j]) : 0.f;
#pragma unroll
                    for (int e = 0; e < V; ++e) acc[t][e] = fmaf(xv, wf[e], acc[t][e]);
                }
            }
        }
        __syncthreads();
        if (active) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < V; ++e) red[((size_t)rg * NT + t) * p.cols_per_cta + tc * V + e] = acc[t][e];
        }
        __syncthreads();
        for (int i = threadIdx.x; i < NT * ncols; i += kThreads) {
            const int t = i / ncols, c = i - t * ncols;
            if (t < nt) {
                float s = 0.f;
                for (int g = 0; g < rg_n; ++g) s += red[((size_t)g * NT + t) * p.cols_per_cta + c];
                p.part[((size_t)blockIdx.x * p.n + t0 + t) * p.r + blockIdx.y * p.cols_per_cta + c] = s;
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.tickets[blockIdx.y], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < p.n * ncols; i += kThreads) {
        const int t = i / ncols, c = blockIdx.y * p.cols_per_cta + (i - t * ncols);
        float s = 0.f;
        for (int sp = 0; sp < (int)gridDim.x; ++sp) s += __ldcg(&p.part[((size_t)sp * p.n + t) * p.r + c]);
        p.u[(size_t)t * p.r + c] = s;
    }
    if (threadIdx.x == 0) p.tickets[blockIdx.y] = 0u;
}

// ---------------------------------------------------------------------------
// Host launchers.

size_t gate_smem_bytes(int /*wdtype*/, int nt, int d, int r, int gate_kind, int cpb, int mw) {
    return gate_smem_layout(nt, d, r, gate_kind, cpb, mw).total;
}

template <class T, int NT, int RW, int GATE>
static cudaError_t launch_gate_t(const GateParams& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
    auto kern = k_gate<T, NT, RW, GATE>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(kThreads), smem, s, pdl, p);
}

template <class T, int NT>
static cudaError_t launch_gate_nt(const GateParams& p, int rw, int gate_kind, int grid, size_t smem,
                                  cudaStream_t s, bool pdl) {
    if (gate_kind == kGatePreselected) return launch_gate_t<T, NT, 1, kGatePreselected>(p, grid, smem, s, pdl);
    if (gate_kind == kGateLopa)
        return rw == 4 ? launch_gate_t<T, NT, 4, kGateLopa>(p, grid, smem, s, pdl)
                       : launch_gate_t<T, NT, 1, kGateLopa>(p, grid, smem, s, pdl);
    return rw == 4 ? launch_gate_t<T, NT, 4, kGateDense>(p, grid, smem, s, pdl)
                   : launch_gate_t<T, NT, 1, kGateDense>(p, grid, smem, s, pdl);
}

template <class T>
static cudaError_t launch_gate_dt(const GateParams& p, int nt, int rw, int gate_kind, int grid,
                                  size_t smem, cudaStream_t s, bool pdl) {
    switch (nt) {
        case 1: return launch_gate_nt<T, 1>(p, rw, gate_kind, grid, smem, s, pdl);
        case 2: return launch_gate_nt<T, 2>(p, rw, gate_kind, grid, smem, s, pdl);
        case 4: return launch_gate_nt<T, 4>(p, rw, gate_kind, grid, smem, s, pdl);
        case 8: return launch_gate_nt<T, 8>(p, rw, gate_kind, grid, smem, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gate(int wdtype, const GateParams& p, int nt, int rw, int gate_kind, int grid,
                        size_t smem, cudaStream_t s, bool pdl) {
    return wdtype == 0 ? launch_gate_dt<bf16>(p, nt, rw, gate_kind, grid, smem, s, pdl)
                       : launch_gate_dt<float>(p, nt, rw, gate_kind, grid, smem, s, pdl);
}

template <class T, int NT>
static cudaError_t launch_lopa_u_t(const LopaUParams& p, dim3 grid, cudaStream_t s, bool pdl) {
    constexpr int V = Elem<T>::kVec;
    const int rg_n = kThreads / (p.cols_per_cta / V);
    const size_t smem = (size_t)rg_n * NT * p.cols_per_cta * sizeof(float);
    auto kern = k_lopa_u<T, NT>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, grid, dim3(kThreads), smem, s, pdl, p);
}

cudaError_t launch_lopa_u(int wdtype, const LopaUParams& p, int nt, dim3 grid, cudaStream_t s, bool pdl) {
    if (wdtype == 0) {
        switch (nt) {
            case 1: return launch_lopa_u_t<bf16, 1>(p, grid, s, pdl);
            case 2: return launch_lopa_u_t<bf16, 2>(p, grid, s, pdl);
            case 4: return launch_lopa_u_t<bf16, 4>(p, grid, s, pdl);
            default: return launch_lopa_u_t<bf16, 8>(p, grid, s, pdl);
        }
    }
    switch (nt) {
        case 1: return launch_lopa_u_t<float, 1>(p, grid, s, pdl);
        case 2: return launch_lopa_u_t<float, 2>(p, grid, s, pdl);
        case 4: return launch_lopa_u_t<float, 4>(p, grid, s, pdl);
        default: return launch_lopa_u_t<float, 8>(p, grid, s, pdl);
    }
}

}  // namespace sffn
