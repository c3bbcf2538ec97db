// Gate-first kernels.
//
// k_gate_stream (dense or LoPA gate): a CTA owns the contiguous channel range
// [c0, c0 + cpb); each warp owns a contiguous block of those rows and streams
// them through its own ring of shared-memory pieces filled by 1-D bulk copies
// (TMA engine, mbarrier completion, L2 evict-first).  The first pieces are
// issued before the programmatic-launch wait: weights never depend on an
// earlier kernel.  Per channel:
//   1. gate   z[t,k] = <x_t, W_gate[:,k]> (row of d) or <u_t, B[:,k]> (LoPA, row of r);
//   2. select active iff z > tau -- "Model Casting and Low-Parameter Gating"
//             (abstract): the gate is evaluated first and only channels whose
//             activation is non-zero go on;
//   3. up     for a channel active in any token, h[k][t] = (z - tau) <x_t, W_up[:,k]>
//             (0 for tokens that did not select k); only active W_up rows are
//             read ("Mixture-of-Channels", section "Dentro il mixture");
//   4. list   ordered compaction of the CTA's active channels into its own
//             fixed slot range (block-wide prefix sum): an ascending list with
//             no global atomics.
// The dense FFN (force_all) streams the W_up rows too, interleaved with the gate
// pieces.  In the z-only mode (top-K) the kernel stops after step 1.
//
// k_gate_presel: the up pass after top-K, reading the selection back.
//
// k_lopa_u: LoPA's first stage u = x A ("Model Casting and Low-Parameter
// Gating", abstract: a low-FLOPs parameterization of the gating matrix, read as
// the rank-r product A B).  A split-d grid writes partial sums; the last CTA of
// each column group (ticket counter) adds them in split order.
#include "common.cuh"

namespace sffn {

constexpr int kStashRows = 16;   // rows per streamed piece, at most

// Shared-memory x (and LoPA u) rows are fp32.  For 8-wide (bf16) chunks a row
// of `len` floats holds the first halves of all chunks, then the second
// halves, so consecutive lanes' 16-byte reads hit consecutive banks.
template <int V>
__device__ __forceinline__ int xpos(int len, int c, int e) {
    if (V == 8) return e < 4 ? c * 4 + e : (len >> 1) + c * 4 + (e - 4);
    return c * 4 + e;
}

// <16-byte weight chunk, x chunk c of one token row in shared memory>, added
// into two accumulators (even and odd elements) to halve the FMA chain.
template <class WT>
__device__ __forceinline__ void chunk_dot(const uint4& w, const float* xrow, int len, int c, float& a0,
                                          float& a1) {
    constexpr int V = Elem<WT>::kVec;
    float wf[V];
    unpack<WT>(w, wf);
    const float4 a = *reinterpret_cast<const float4*>(xrow + xpos<V>(len, c, 0));
    a0 = fmaf(wf[0], a.x, a0);
    a1 = fmaf(wf[1], a.y, a1);
    a0 = fmaf(wf[2], a.z, a0);
    a1 = fmaf(wf[3], a.w, a1);
    if (V == 8) {
        const float4 b = *reinterpret_cast<const float4*>(xrow + xpos<V>(len, c, 4));
        a0 = fmaf(wf[4], b.x, a0);
        a1 = fmaf(wf[5], b.y, a1);
        a0 = fmaf(wf[6], b.z, a0);
        a1 = fmaf(wf[7], b.w, a1);
    }
}

// Stage tokens [t0, t0 + nt) of a global row-major n x len array (type XT) as
// fp32 rows of `len` in shared memory (chunk layout of weight type WT); rows
// nt..NT-1 are zero.  16-byte loads, all of a thread's loads issued before any
// store (a handful of round trips at most).  All threads of the block take part.
template <class WT, class XT, int NT>
__device__ __forceinline__ void stage_rows(float* dst, const XT* src, int len, int t0, int nt) {
    constexpr int V = Elem<WT>::kVec;
    constexpr int XV = 16 / sizeof(XT);                 // elements per 16-byte load
    constexpr int U = 4;
    const int per_row = len / XV;                        // len is a multiple of 8
    const int total = NT * per_row;
    for (int base = threadIdx.x; base < total; base += U * blockDim.x) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            const int t = i / per_row;
            v[u] = (i < total && t < nt)
                       ? *reinterpret_cast<const uint4*>(src + (size_t)(t0 + t) * len + (size_t)(i - t * per_row) * XV)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            if (i < total) {
                const int t = i / per_row, j0 = (i - t * per_row) * XV;
                float f[XV];
                unpack<XT>(v[u], f);
#pragma unroll
                for (int e = 0; e < XV; ++e) {
                    const int j = j0 + e;
                    dst[t * len + xpos<V>(len, j / V, j % V)] = f[e];
                }
            }
        }
    }
}

// acc[t] = <row, x_t> over a global row of cpr 16-byte chunks, read with
// L1-bypassing loads (16 in flight per lane); every lane ends with the sums.
template <class WT, int NT>
__device__ __forceinline__ void warp_dot_global(const WT* __restrict__ row, int cpr, const float* xs, int len,
                                                float (&acc)[NT]) {
    constexpr int UB = NT >= 4 ? 8 : 16;
    const int lane = threadIdx.x & 31;
    float acc1[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = acc1[t] = 0.f;
    for (int cb = lane; cb < cpr; cb += 32 * UB) {
        uint4 wv[UB];
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            const int c = cb + 32 * u;
            wv[u] = c < cpr ? ld_stream(row + (size_t)c * Elem<WT>::kVec) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            const int c = cb + 32 * u;
            if (c < cpr) {
#pragma unroll
                for (int t = 0; t < NT; ++t) chunk_dot<WT>(wv[u], xs + t * len, len, c, acc[t], acc1[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = warp_sum(acc[t] + acc1[t]);
}

// Per-lane partial of <piece, x_t> over chunks [0, nch) of a shared-memory
// piece whose chunk 0 is chunk `coff` of the row.
template <class WT, int NT>
__device__ __forceinline__ void piece_dot(const unsigned char* piece, int nch, int coff, const float* xs, int len,
                                          float (&acc)[NT], float (&acc1)[NT]) {
    const int lane = threadIdx.x & 31;
#pragma unroll 2
    for (int c = lane; c < nch; c += 32) {
        const uint4 w = reinterpret_cast<const uint4*>(piece)[c];
#pragma unroll
        for (int t = 0; t < NT; ++t) chunk_dot<WT>(w, xs + t * len, len, coff + c, acc[t], acc1[t]);
    }
}

// ---------------------------------------------------------------------------

struct StreamSmem {
    size_t xs, us, stash, mask, flag, scan, bars, bufs, total;
};
__host__ __device__ inline StreamSmem stream_smem_layout(int nt, int d, int r, int gate_kind, int cpb, int mw,
                                                         int sb, int nb) {
    StreamSmem L;
    size_t o = 0;
    L.xs = o;    o += (size_t)nt * d * sizeof(float);
    L.us = o;    o += gate_kind == kGateLopa ? (size_t)nt * r * sizeof(float) : 0;
    L.stash = o; o += (size_t)kWarps * kStashRows * nt * sizeof(float);
    L.mask = o;  o += (size_t)cpb * mw * sizeof(uint32_t);
    L.flag = o;  o += ((size_t)cpb + 15) & ~(size_t)15;
    L.scan = o;  o += 48 * sizeof(int);
    o = (o + 15) & ~(size_t)15;                      // mbarriers need 8-byte alignment
    L.bars = o;  o += (size_t)kWarps * nb * sizeof(uint64_t);
    o = (o + 127) & ~(size_t)127;
    L.bufs = o;  o += (size_t)kWarps * nb * sb;
    L.total = o;
    return L;
}

template <class T, int NT, int GATE>
__global__ void __launch_bounds__(kThreads, 2) k_gate_stream(const GateParams p) {
    constexpr int V = Elem<T>::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * p.cpb;
    const int nslots = max(0, min(p.cpb, p.d_ff - c0));
    const StreamSmem L = stream_smem_layout(NT, p.d, p.r, GATE, p.cpb, p.mw, p.sb, p.nb);
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    float* us = reinterpret_cast<float*>(smem + L.us);
    float* stash = reinterpret_cast<float*>(smem + L.stash) + warp * kStashRows * NT;
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + L.mask);
    uint8_t* flag = reinterpret_cast<uint8_t*>(smem + L.flag);
    int* scan_sh = reinterpret_cast<int*>(smem + L.scan);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * p.nb;
    unsigned char* bufs = smem + L.bufs + (size_t)warp * p.nb * p.sb;

    const int glen = GATE == kGateLopa ? p.r : p.d;               // gate row length
    const float* gx = GATE == kGateLopa ? us : xs;                  // what the gate row multiplies
    const int rb = glen * (int)sizeof(T);
    const int cpr = glen / V;
    const bool alt = p.force_all && GATE == kGateDense && p.out == kOutSelectUp;
    const T* wup = static_cast<const T*>(p.wup);
    const char* gbase = reinterpret_cast<const char*>(static_cast<const T*>(GATE == kGateLopa ? p.bcm : p.wg) +
                                                      (size_t)c0 * glen);
    const char* ubase = reinterpret_cast<const char*>(wup + (size_t)c0 * p.d);
    const int wr0 = (int)((long long)nslots * warp / kWarps);
    const int nrows = (int)((long long)nslots * (warp + 1) / kWarps) - wr0;
    int rpp, ppr, pb;
    if (rb <= p.sb) {
        rpp = min(p.sb / rb, kStashRows);
        ppr = 1;
        pb = rpp * rb;
    } else {
        rpp = 1;
        ppr = (rb + p.sb - 1) / p.sb;
        pb = ((rb + ppr - 1) / ppr + 15) & ~15;
    }
    const int gpieces = rb <= p.sb ? (nrows + rpp - 1) / rpp : nrows * ppr;
    const int ppt = alt ? 2 * gpieces : gpieces;
    const int ntiles = (p.n + NT - 1) / NT;
    const int total = ppt * ntiles;
    const uint64_t pol = l2_evict_first();

    auto issue = [&](int i) {
        const int ip = i % ppt;
        const int j = alt ? ip >> 1 : ip;
        const char* base = ((alt && (ip & 1)) ? ubase : gbase) + (size_t)wr0 * rb;
        uint32_t bytes;
        const char* src;
        if (rb <= p.sb) {
            const int r0 = j * rpp;
            bytes = (uint32_t)(min(rpp, nrows - r0) * rb);
            src = base + (size_t)r0 * rb;
        } else {
            const int row = j / ppr, off = (j - row * ppr) * pb;
            bytes = (uint32_t)min(pb, rb - off);
            src = base + (size_t)row * rb + off;
        }
        uint64_t* bar = bars + (i % p.nb);
        mbar_expect_tx(bar, bytes);
        bulk_load(bufs + (size_t)(i % p.nb) * p.sb, src, bytes, bar, pol);
    };

    if (lane == 0) {
        for (int b = 0; b < p.nb; ++b) mbar_init(bars + b, 1);
        fence_mbar_init();
        for (int i = 0; i < min(p.nb, total); ++i) issue(i);
    }
    __syncwarp();

    griddep_wait();
    griddep_launch_dependents();

    for (int i = threadIdx.x; i < p.cpb; i += kThreads) flag[i] = 0;
    for (int i = threadIdx.x; i < p.cpb * p.mw; i += kThreads) smask[i] = 0u;

    // z -> selection -> (maybe) up -> h, for slot s of this CTA.  u_in: the up
    // dot when it was streamed (alt), else it is fetched here.
    auto finish = [&](int s, const float (&z)[NT], const float* u_in, int t0, int nt) {
        const int k = c0 + s;
        if (p.out == kOutWriteZ) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == t && t < nt) p.zbuf[(size_t)(t0 + t) * p.d_ff + k] = z[t];
            return;
        }
        uint32_t tokmask = 0u;
#pragma unroll
        for (int t = 0; t < NT; ++t) tokmask |= (t < nt && z[t] > p.tau ? 1u : 0u) << t;
        if (tokmask != 0u || p.force_all) {
            float u[NT];
            if (u_in) {
#pragma unroll
                for (int t = 0; t < NT; ++t) u[t] = u_in[t];
            } else {
                warp_dot_global<T, NT>(wup + (size_t)k * p.d, p.d / V, xs, p.d, u);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == t && t < nt)
                    p.lst_h[(size_t)k * p.n + t0 + t] = ((tokmask >> t) & 1u) ? (z[t] - p.tau) * u[t] : 0.f;
            if (lane == 0) {
                flag[s] = 1;
                smask[s * p.mw + (t0 >> 5)] |= tokmask << (t0 & 31);
            }
        } else if (ntiles > 1) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == t && t < nt) p.lst_h[(size_t)k * p.n + t0 + t] = 0.f;
        }
    };

    bool abort = false;
    int abort_at = 0;
    int i = 0;
    for (int tile = 0; tile < ntiles; ++tile) {
        const int t0 = tile * NT;
        const int nt = min(NT, p.n - t0);
        __syncthreads();
        stage_rows<T, T, NT>(xs, static_cast<const T*>(p.x), p.d, t0, nt);
        if (GATE == kGateLopa) stage_rows<T, float, NT>(us, p.u, p.r, t0, nt);
        __syncthreads();
        float accz[NT], accu[NT], accz1[NT], accu1[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) accz[t] = accu[t] = accz1[t] = accu1[t] = 0.f;
        for (int ip = 0; ip < ppt; ++ip, ++i) {
            if (abort) continue;
            if (!mbar_wait_warp(bars + (i % p.nb), (uint32_t)((i / p.nb) & 1))) {
                abort = true;
                abort_at = i;
                if (lane == 0) atomicOr(p.status, (int)kStatusWaitTimeout);
                continue;
            }
            const unsigned char* buf = bufs + (size_t)(i % p.nb) * p.sb;
            const int j = alt ? ip >> 1 : ip;
            const bool up_piece = alt && (ip & 1);
            if (rb <= p.sb) {
                const int r0 = j * rpp, cnt = min(rpp, nrows - r0);
                for (int q = 0; q < cnt; ++q) {
                    float v[NT], v1[NT];
#pragma unroll
                    for (int t = 0; t < NT; ++t) v[t] = v1[t] = 0.f;
                    piece_dot<T, NT>(buf + (size_t)q * rb, cpr, 0, up_piece ? xs : gx, up_piece ? p.d : glen, v,
                                     v1);
#pragma unroll
                    for (int t = 0; t < NT; ++t) v[t] = warp_sum(v[t] + v1[t]);
                    const int s = wr0 + r0 + q;
                    if (!alt) {
                        finish(s, v, nullptr, t0, nt);
                    } else if (!up_piece) {
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            if (lane == t) stash[q * NT + t] = v[t];
                    } else {
                        float z[NT];
#pragma unroll
                        for (int t = 0; t < NT; ++t) z[t] = stash[q * NT + t];
                        finish(s, z, v, t0, nt);
                    }
                }
            } else {
                const int row = j / ppr, part = j - row * ppr, off = part * pb;
                const int nch = min(pb, rb - off) / 16;
                if (up_piece) piece_dot<T, NT>(buf, nch, off / 16, xs, p.d, accu, accu1);
                else piece_dot<T, NT>(buf, nch, off / 16, gx, glen, accz, accz1);
                if (part == ppr - 1 && (up_piece || !alt)) {
                    float z[NT], u[NT];
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        z[t] = warp_sum(accz[t] + accz1[t]);
                        u[t] = warp_sum(accu[t] + accu1[t]);
                        accz[t] = accu[t] = accz1[t] = accu1[t] = 0.f;
                    }
                    finish(wr0 + row, z, alt ? u : nullptr, t0, nt);
                }
            }
            __syncwarp();
            if (lane == 0 && i + p.nb < total) {
                fence_proxy_async();
                issue(i + p.nb);
            }
        }
    }
    if (abort) {
        // Pieces [abort_at, abort_at + nb) were issued and not consumed: give each
        // a bounded wait so no copy lands after the CTA has gone.
        for (int q = abort_at; q < min(abort_at + p.nb, total); ++q)
            mbar_wait_warp(bars + (q % p.nb), (uint32_t)((q / p.nb) & 1));
    }
    if (p.out == kOutWriteZ) return;

    __syncthreads();
    const int per = (nslots + kThreads - 1) / kThreads;
    const int sb0 = threadIdx.x * per;
    int cnt = 0;
    for (int q = 0; q < per; ++q)
        if (sb0 + q < nslots && flag[sb0 + q]) ++cnt;
    int tot = 0;
    int pos = block_exclusive_scan(cnt, &tot, scan_sh);
    for (int q = 0; q < per; ++q) {
        const int s = sb0 + q;
        if (s < nslots && flag[s]) {
            p.lst_idx[c0 + pos] = c0 + s;
            for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + s) * p.mw + w] = smask[s * p.mw + w];
            ++pos;
        }
    }
    if (threadIdx.x == 0) p.seg_count[blockIdx.x] = tot;
}

// ---------------------------------------------------------------------------
// Up pass after top-K: the selection (sel, gbuf) is read back per channel and
// the selected channels' W_up rows are read with 16-byte loads.

struct PreselSmem {
    size_t xs, mask, flag, scan, total;
};
__host__ __device__ inline PreselSmem presel_smem_layout(int nt, int d, int cpb, int mw) {
    PreselSmem L;
    size_t o = 0;
    L.xs = o;   o += (size_t)nt * d * sizeof(float);
    L.mask = o; o += (size_t)cpb * mw * sizeof(uint32_t);
    L.flag = o; o += ((size_t)cpb + 15) & ~(size_t)15;
    L.scan = o; o += 48 * sizeof(int);
    L.total = o;
    return L;
}

template <class T, int NT>
__global__ void __launch_bounds__(kThreads, 2) k_gate_presel(const GateParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int V = Elem<T>::kVec;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * p.cpb;
    const int nslots = max(0, min(p.cpb, p.d_ff - c0));
    const PreselSmem L = presel_smem_layout(NT, p.d, p.cpb, p.mw);
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + L.mask);
    uint8_t* flag = reinterpret_cast<uint8_t*>(smem + L.flag);
    int* scan_sh = reinterpret_cast<int*>(smem + L.scan);
    const T* wup = static_cast<const T*>(p.wup);
    const int ntiles = (p.n + NT - 1) / NT;

    griddep_wait();
    griddep_launch_dependents();

    for (int i = threadIdx.x; i < p.cpb; i += kThreads) flag[i] = 0;
    for (int i = threadIdx.x; i < p.cpb * p.mw; i += kThreads) smask[i] = 0u;

    for (int tile = 0; tile < ntiles; ++tile) {
        const int t0 = tile * NT;
        const int nt = min(NT, p.n - t0);
        __syncthreads();
        stage_rows<T, T, NT>(xs, static_cast<const T*>(p.x), p.d, t0, nt);
        __syncthreads();
        for (int s = warp; s < nslots; s += kWarps) {
            const int k = c0 + s;
            uint32_t tokmask = 0u;
            float gv[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                gv[t] = 0.f;
                if (t < nt) {
                    const size_t o = (size_t)(t0 + t) * p.d_ff + k;
                    if (p.sel[o]) {
                        tokmask |= 1u << t;
                        gv[t] = p.gbuf[o];
                    }
                }
            }
            if (tokmask != 0u || p.force_all) {
                float u[NT];
                warp_dot_global<T, NT>(wup + (size_t)k * p.d, p.d / V, xs, p.d, u);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (lane == t && t < nt)
                        p.lst_h[(size_t)k * p.n + t0 + t] = ((tokmask >> t) & 1u) ? gv[t] * u[t] : 0.f;
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
    __syncthreads();
    const int per = (nslots + kThreads - 1) / kThreads;
    const int sb0 = threadIdx.x * per;
    int cnt = 0;
    for (int q = 0; q < per; ++q)
        if (sb0 + q < nslots && flag[sb0 + q]) ++cnt;
    int tot = 0;
    int pos = block_exclusive_scan(cnt, &tot, scan_sh);
    for (int q = 0; q < per; ++q) {
        const int s = sb0 + q;
        if (s < nslots && flag[s]) {
            p.lst_idx[c0 + pos] = c0 + s;
            for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + s) * p.mw + w] = smask[s * p.mw + w];
            ++pos;
        }
    }
    if (threadIdx.x == 0) p.seg_count[blockIdx.x] = tot;
}

// ---------------------------------------------------------------------------
// LoPA stage 1: u[t][j] = <x_t, A[:, j]>, with A stored transposed so column j
// of A is one contiguous row.  kLopaRowsPerCta rows per CTA, each split over
// kWarps / kLopaRowsPerCta warps; every lane keeps up to 16 chunk loads in
// flight.  The rows are bulk-prefetched into L2 before the programmatic-launch
// wait (weights never depend on an earlier kernel); u needs no cross-CTA sum.

template <class T, int NT>
__global__ void __launch_bounds__(kThreads) k_lopa_u(const LopaUParams p) {
    constexpr int V = Elem<T>::kVec;
    constexpr int RPC = kLopaRowsPerCta;
    constexpr int WPR = kWarps / RPC;            // warps per row
    constexpr int TPR = WPR * 32;                // threads per row
    constexpr int UB = NT >= 8 ? 2 : 16 / (2 * NT) > 0 ? 16 / (2 * NT) : 1;
    __shared__ float red[RPC][WPR][NT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rr = warp / WPR, wq = warp - rr * WPR;
    const int j = blockIdx.x * RPC + rr;
    const bool ok = j < p.r;
    const int cpr = p.d / V;
    const int tr = wq * 32 + lane;
    const T* row = static_cast<const T*>(p.at) + (size_t)(ok ? j : 0) * p.d;
    const T* x = static_cast<const T*>(p.x);
    if (ok && tr == 0) bulk_prefetch_l2(row, (uint32_t)(p.d * sizeof(T)));

    griddep_wait();
    griddep_launch_dependents();

    for (int t0 = 0; t0 < p.n; t0 += NT) {
        const int nt = min(NT, p.n - t0);
        float a0[NT], a1[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) a0[t] = a1[t] = 0.f;
        for (int cb = tr; cb < cpr; cb += UB * TPR) {
            uint4 w[UB], xv[UB][NT];
#pragma unroll
            for (int u = 0; u < UB; ++u) {
                const int c = cb + u * TPR;
                const bool in = ok && c < cpr;
                w[u] = in ? ld_stream(row + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    xv[u][t] = (in && t < nt) ? *reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * p.d + (size_t)c * V)
                                              : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < UB; ++u) {
                float wf[V];
                unpack<T>(w[u], wf);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    float xf[V];
                    unpack<T>(xv[u][t], xf);
#pragma unroll
                    for (int e = 0; e < V; e += 2) {
                        a0[t] = fmaf(wf[e], xf[e], a0[t]);
                        a1[t] = fmaf(wf[e + 1], xf[e + 1], a1[t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(a0[t] + a1[t]);
            if (lane == 0) red[rr][wq][t] = v;
        }
        __syncthreads();
        if ((int)threadIdx.x < RPC * NT) {
            const int r2 = threadIdx.x / NT, t = threadIdx.x - r2 * NT;
            const int jj = blockIdx.x * RPC + r2;
            if (jj < p.r && t < nt) {
                float s = 0.f;
#pragma unroll
                for (int q = 0; q < WPR; ++q) s += red[r2][q][t];
                p.u[(size_t)(t0 + t) * p.r + jj] = s;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Host launchers.

size_t gate_smem_bytes(int /*wdtype*/, int nt, int d, int /*r*/, int /*gate_kind*/, int cpb, int mw) {
    return presel_smem_layout(nt, d, cpb, mw).total;
}

size_t gate_stream_smem_bytes(int nt, int d, int r, int gate_kind, int cpb, int mw, int sb, int nb) {
    return stream_smem_layout(nt, d, r, gate_kind, cpb, mw, sb, nb).total;
}

template <class T, int NT>
static cudaError_t launch_presel_t(const GateParams& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
    auto kern = k_gate_presel<T, NT>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(kThreads), smem, s, pdl, p);
}

template <class T>
static cudaError_t launch_presel_dt(const GateParams& p, int nt, int grid, size_t smem, cudaStream_t s, bool pdl) {
    switch (nt) {
        case 1: return launch_presel_t<T, 1>(p, grid, smem, s, pdl);
        case 2: return launch_presel_t<T, 2>(p, grid, smem, s, pdl);
        case 4: return launch_presel_t<T, 4>(p, grid, smem, s, pdl);
        case 8: return launch_presel_t<T, 8>(p, grid, smem, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gate(int wdtype, const GateParams& p, int nt, int /*rw*/, int gate_kind, int grid,
                        size_t smem, cudaStream_t s, bool pdl) {
    if (gate_kind != kGatePreselected) return cudaErrorInvalidValue;
    return wdtype == 0 ? launch_presel_dt<bf16>(p, nt, grid, smem, s, pdl)
                       : launch_presel_dt<float>(p, nt, grid, smem, s, pdl);
}

template <class T, int NT, int GATE>
static cudaError_t launch_stream_t(const GateParams& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
    auto kern = k_gate_stream<T, NT, GATE>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(kThreads), smem, s, pdl, p);
}

template <class T, int NT>
static cudaError_t launch_stream_nt(const GateParams& p, int gate_kind, int grid, size_t smem, cudaStream_t s,
                                    bool pdl) {
    return gate_kind == kGateLopa ? launch_stream_t<T, NT, kGateLopa>(p, grid, smem, s, pdl)
                                  : launch_stream_t<T, NT, kGateDense>(p, grid, smem, s, pdl);
}

template <class T>
static cudaError_t launch_stream_dt(const GateParams& p, int nt, int gate_kind, int grid, size_t smem,
                                    cudaStream_t s, bool pdl) {
    switch (nt) {
        case 1: return launch_stream_nt<T, 1>(p, gate_kind, grid, smem, s, pdl);
        case 2: return launch_stream_nt<T, 2>(p, gate_kind, grid, smem, s, pdl);
        case 4: return launch_stream_nt<T, 4>(p, gate_kind, grid, smem, s, pdl);
        case 8: return launch_stream_nt<T, 8>(p, gate_kind, grid, smem, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gate_stream(int wdtype, const GateParams& p, int nt, int gate_kind, int grid, size_t smem,
                               cudaStream_t s, bool pdl) {
    if (gate_kind == kGatePreselected || p.sb <= 0 || p.sb % 16 || p.nb <= 0) return cudaErrorInvalidValue;
    return wdtype == 0 ? launch_stream_dt<bf16>(p, nt, gate_kind, grid, smem, s, pdl)
                       : launch_stream_dt<float>(p, nt, gate_kind, grid, smem, s, pdl);
}

template <class T, int NT>
static cudaError_t launch_lopa_u_t(const LopaUParams& p, cudaStream_t s, bool pdl) {
    const int grid = (p.r + kLopaRowsPerCta - 1) / kLopaRowsPerCta;
    return launch_ex(k_lopa_u<T, NT>, dim3(grid), dim3(kThreads), 0, s, pdl, p);
}

cudaError_t launch_lopa_u(int wdtype, const LopaUParams& p, int nt, cudaStream_t s, bool pdl) {
    if (wdtype == 0) {
        switch (nt) {
            case 1: return launch_lopa_u_t<bf16, 1>(p, s, pdl);
            case 2: return launch_lopa_u_t<bf16, 2>(p, s, pdl);
            case 4: return launch_lopa_u_t<bf16, 4>(p, s, pdl);
            default: return launch_lopa_u_t<bf16, 8>(p, s, pdl);
        }
    }
    switch (nt) {
        case 1: return launch_lopa_u_t<float, 1>(p, s, pdl);
        case 2: return launch_lopa_u_t<float, 2>(p, s, pdl);
        case 4: return launch_lopa_u_t<float, 4>(p, s, pdl);
        default: return launch_lopa_u_t<float, 8>(p, s, pdl);
    }
}

}  // namespace sffn
