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
#include "dot.cuh"

namespace sffn {

constexpr int kStreamWarps = 16;  // warps of a streaming gate CTA (one CTA per SM)
constexpr int kStreamThreads = kStreamWarps * 32;

// ---------------------------------------------------------------------------

struct StreamSmem {
    size_t xs, us, zpart, zfin, wl, mask, flag, scan, bars, bufs, total;
};
// zparts: partial gate dots per (slot, part), see k_gate_stream.
__host__ __device__ inline StreamSmem stream_smem_layout(int nt, int d, int r, int gate_kind, int cpb, int mw,
                                                         int sb, int nb) {
    StreamSmem L;
    const int glen = gate_kind == kGateLopa ? r : d;
    const int rb = glen * 4;                      // worst case (fp32 rows) for the part count
    const int ppr = rb <= sb ? 1 : (rb + sb - 1) / sb + 1;
    size_t o = 0;
    L.xs = o;    o += (size_t)nt * d * sizeof(float);
    L.us = o;    o += gate_kind == kGateLopa ? (size_t)nt * r * sizeof(float) : 0;
    L.zpart = o; o += (size_t)cpb * ppr * nt * sizeof(float);
    L.zfin = o;  o += (size_t)cpb * nt * sizeof(float);
    L.wl = o;    o += (size_t)cpb * sizeof(int);
    L.mask = o;  o += (size_t)cpb * mw * sizeof(uint32_t);
    L.flag = o;  o += ((size_t)cpb + 15) & ~(size_t)15;
    L.scan = o;  o += 48 * sizeof(int);
    o = (o + 15) & ~(size_t)15;                      // mbarriers need 8-byte alignment
    L.bars = o;  o += (size_t)kStreamWarps * nb * sizeof(uint64_t);
    o = (o + 127) & ~(size_t)127;
    L.bufs = o;  o += (size_t)kStreamWarps * nb * sb;
    L.total = o;
    return L;
}

// Two phases per token tile.
//  Streaming: the CTA's gate rows are cut into pieces (whole rows, or equal
//  parts of a row); warp w takes a contiguous, balanced range of pieces and
//  streams it through its own ring of bulk copies; each piece leaves its
//  per-token dot product (of whole rows, or a part of a row) in shared memory.
//  No data-dependent work happens here, so every warp keeps streaming.
//  Finish (after a barrier): z = the sum of a row's parts in part order;
//  select; prefetch the active channels' W_down rows into L2; spread the rows
//  that need an up dot evenly over the warps (all their loads in flight at
//  once); h = (z - tau) u.  The dense FFN (force_all) takes the up dot of every
//  row.  Finally the CTA's active channels are compacted into its list segment.
template <class T, int NT, int GATE>
__global__ void __launch_bounds__(kStreamThreads, 1) k_gate_stream(const GateParams p) {
    constexpr int V = Elem<T>::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * p.cpb;
    const int nslots = max(0, min(p.cpb, p.d_ff - c0));
    const StreamSmem L = stream_smem_layout(NT, p.d, p.r, GATE, p.cpb, p.mw, p.sb, p.nb);
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    float* us = reinterpret_cast<float*>(smem + L.us);
    float* zpart = reinterpret_cast<float*>(smem + L.zpart);
    float* zfin = reinterpret_cast<float*>(smem + L.zfin);
    int* wl = reinterpret_cast<int*>(smem + L.wl);
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + L.mask);
    uint8_t* flag = reinterpret_cast<uint8_t*>(smem + L.flag);
    int* scan_sh = reinterpret_cast<int*>(smem + L.scan);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * p.nb;
    unsigned char* bufs = smem + L.bufs + (size_t)warp * p.nb * p.sb;

    const int glen = GATE == kGateLopa ? p.r : p.d;               // gate row length
    const float* gx = GATE == kGateLopa ? us : xs;                  // what the gate row multiplies
    const int rb = glen * (int)sizeof(T);
    const int cpr = glen / V;
    const T* wup = static_cast<const T*>(p.wup);
    const char* gbase = reinterpret_cast<const char*>(static_cast<const T*>(GATE == kGateLopa ? p.bcm : p.wg) +
                                                      (size_t)c0 * glen);
    // pieces: rpp whole rows each, or ppr parts of one row (pb bytes, the last shorter)
    int rpp, ppr, pb;
    if (rb <= p.sb) {
        const int per_warp = (nslots + kStreamWarps - 1) / kStreamWarps;
        rpp = max(1, min(p.sb / rb, per_warp));
        ppr = 1;
        pb = rpp * rb;
    } else {
        rpp = 1;
        ppr = (rb + p.sb - 1) / p.sb;
        pb = ((rb + ppr - 1) / ppr + 15) & ~15;
        ppr = (rb + pb - 1) / pb;
    }
    const int npieces = rb <= p.sb ? (nslots + rpp - 1) / rpp : nslots * ppr;   // per tile
    const int w0 = (int)((long long)npieces * warp / kStreamWarps);
    const int wcount = (int)((long long)npieces * (warp + 1) / kStreamWarps) - w0;
    const int ntiles = (p.n + NT - 1) / NT;
    const int total = wcount * ntiles;
    const uint64_t pol = l2_evict_first();

    // Cursor over this warp's pieces: (g, part) of piece w0 + j, ring slot and parity.
    struct Cursor {
        int j, g, part, buf, parity;
    };
    auto start_of = [&](Cursor& c) {
        c.j = 0;
        c.g = rb <= p.sb ? w0 : w0 / ppr;
        c.part = rb <= p.sb ? 0 : w0 - c.g * ppr;
    };
    auto advance = [&](Cursor& c) {
        if (++c.buf == p.nb) {
            c.buf = 0;
            c.parity ^= 1;
        }
        if (++c.j == wcount) {
            start_of(c);
        } else if (++c.part >= ppr) {
            c.part = 0;
            ++c.g;
        }
    };
    auto issue = [&](const Cursor& c) {
        uint32_t bytes;
        const char* src;
        if (rb <= p.sb) {
            const int r0 = c.g * rpp;
            bytes = (uint32_t)(min(rpp, nslots - r0) * rb);
            src = gbase + (size_t)r0 * rb;
        } else {
            const int off = c.part * pb;
            bytes = (uint32_t)min(pb, rb - off);
            src = gbase + (size_t)c.g * rb + off;
        }
        uint64_t* bar = bars + c.buf;
        mbar_expect_tx(bar, bytes);
        bulk_load(bufs + (size_t)c.buf * p.sb, src, bytes, bar, pol);
    };

    Cursor ic{0, 0, 0, 0, 0};
    start_of(ic);
    int issued = 0;
    if (lane == 0) {
        for (int b = 0; b < p.nb; ++b) mbar_init(bars + b, 1);
        fence_mbar_init();
    }
    __syncwarp();
    // Weights never depend on an earlier kernel: start streaming before the
    // PDL wait -- one piece per warp only, so that x, read right after the
    // wait, does not queue behind a deep ring of weight traffic.
    if (total > 0) {
        if (lane == 0) issue(ic);
        advance(ic);
        ++issued;
    }
    __syncwarp();

    griddep_wait();
    griddep_launch_dependents();

    for (int i = threadIdx.x; i < p.cpb; i += kStreamThreads) flag[i] = 0;
    for (int i = threadIdx.x; i < p.cpb * p.mw; i += kStreamThreads) smask[i] = 0u;

    bool abort = false;
    int abort_at = 0, consumed = 0;
    Cursor cc{0, 0, 0, 0, 0};
    start_of(cc);
    for (int tile = 0; tile < ntiles; ++tile) {
        const int t0 = tile * NT;
        const int nt = min(NT, p.n - t0);
        __syncthreads();
        stage_rows<T, T, NT>(xs, static_cast<const T*>(p.x), p.d, t0, nt);
        if (GATE == kGateLopa) stage_rows<T, float, NT>(us, p.u, p.r, t0, nt);
        // x is on its way: fill the rest of the ring.
        for (; tile == 0 && issued < min(p.nb, total); ++issued) {
            if (lane == 0) issue(ic);
            advance(ic);
        }
        __syncthreads();

        // ---- streaming phase
        // Rows selected while streaming get their W_up and W_down rows pulled
        // into L2 at once, so the up dots and the down pass read them from L2.
        const bool prefetch_rows = p.out == kOutSelectUp && !p.force_all;
        auto prefetch_active = [&](int k) {
            bulk_prefetch_l2(wup + (size_t)k * p.d, (uint32_t)(p.d * sizeof(T)));
            if (p.wdn)
                bulk_prefetch_l2(static_cast<const T*>(p.wdn) + (size_t)k * p.d, (uint32_t)(p.d * sizeof(T)));
        };
        float zrow[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) zrow[t] = 0.f;
        for (int j = 0; j < wcount; ++j) {
            if (abort) continue;
            if (!mbar_wait_warp(bars + cc.buf, (uint32_t)cc.parity)) {
                abort = true;
                abort_at = consumed;
                if (lane == 0) raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                continue;
            }
            const unsigned char* buf = bufs + (size_t)cc.buf * p.sb;
            if (rb <= p.sb) {
                const int r0 = cc.g * rpp, cnt = min(rpp, nslots - r0);
                for (int q = 0; q < cnt; ++q) {
                    float2 v2[NT];
#pragma unroll
                    for (int t = 0; t < NT; ++t) v2[t] = make_float2(0.f, 0.f);
                    piece_dot<T, NT>(buf + (size_t)q * rb, cpr, 0, gx, glen, v2);
                    bool act = false;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float v = warp_sum(v2[t].x + v2[t].y);
                        if (lane == t) zpart[(r0 + q) * NT + t] = v;
                        act |= t < nt && v > p.tau;
                    }
                    if (act && lane == 0 && prefetch_rows) prefetch_active(c0 + r0 + q);
                }
            } else {
                const int off = cc.part * pb;
                float2 v2[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) v2[t] = make_float2(0.f, 0.f);
                piece_dot<T, NT>(buf, min(pb, rb - off) >> 4, off >> 4, gx, glen, v2);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float v = warp_sum(v2[t].x + v2[t].y);
                    if (lane == t) zpart[(cc.g * ppr + cc.part) * NT + t] = v;
                    zrow[t] = cc.part == 0 ? v : zrow[t] + v;
                }
                // The whole row went through this warp: its z is known now.
                if (cc.part == ppr - 1 && cc.j >= cc.part && prefetch_rows && lane == 0) {
                    bool act = false;
#pragma unroll
                    for (int t = 0; t < NT; ++t) act |= t < nt && zrow[t] > p.tau;
                    if (act) prefetch_active(c0 + cc.g);
                }
            }
            __syncwarp();
            if (issued < total) {
                if (lane == 0) {
                    fence_proxy_async();
                    issue(ic);
                }
                advance(ic);
                ++issued;
            }
            advance(cc);
            ++consumed;
        }
        __syncthreads();

        // ---- finish: z, selection, up dots
        for (int sl = threadIdx.x; sl < nslots; sl += kStreamThreads) {
            const int k = c0 + sl;
            uint32_t tokmask = 0u;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float z = 0.f;
                for (int q = 0; q < ppr; ++q) z += zpart[(sl * ppr + q) * NT + t];
                zfin[sl * NT + t] = z;
                if (t < nt) {
                    if (p.out == kOutWriteZ) p.zbuf[(size_t)(t0 + t) * p.d_ff + k] = z;
                    else if (z > p.tau) tokmask |= 1u << t;
                }
            }
            if (p.out == kOutSelectUp && (tokmask || p.force_all)) {
                // The down pass will read this channel's W_down row: start
                // bringing it into L2 now.
                if (tokmask && !flag[sl] && !p.force_all && p.wdn)
                    bulk_prefetch_l2(static_cast<const T*>(p.wdn) + (size_t)k * p.d, (uint32_t)(p.d * sizeof(T)));
                flag[sl] = 1;
                smask[sl * p.mw + (t0 >> 5)] |= tokmask << (t0 & 31);
            }
            wl[sl] = (int)tokmask;                      // this tile's selection, read back below
        }
        __syncthreads();
        if (p.out == kOutWriteZ) continue;
        // rows needing an up dot in this tile, in order
        int* work = reinterpret_cast<int*>(zpart);     // zpart is free until the next tile
        const int nwork = block_compact(nslots, [&](int sl) { return wl[sl] != 0 || p.force_all; }, work, scan_sh);
        for (int i = warp; i < nwork; i += kStreamWarps) {
            const int sl = work[i], k = c0 + sl;
            const uint32_t tokmask = (uint32_t)wl[sl];
            float u[NT];
            warp_dot_global<T, NT>(wup + (size_t)k * p.d, p.d / V, xs, p.d, u);
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == t && t < nt)
                    p.lst_h[(size_t)k * p.n + t0 + t] =
                        ((tokmask >> t) & 1u) ? (zfin[sl * NT + t] - p.tau) * u[t] : 0.f;
        }
        if (ntiles > 1 && !p.force_all) {
            // channels active in another tile only: h = 0 for this tile's tokens
            for (int i = threadIdx.x; i < nslots * NT; i += kStreamThreads) {
                const int sl = i / NT, t = i - sl * NT;
                if (t < nt && wl[sl] == 0) p.lst_h[(size_t)(c0 + sl) * p.n + t0 + t] = 0.f;
            }
        }
        __syncthreads();
    }
    if (abort) {
        // Pieces [abort_at, issued) were issued and not consumed: give each a
        // bounded wait so no copy lands after the CTA has gone.
        for (int q = abort_at; q < issued; ++q)
            mbar_wait_warp(bars + (q % p.nb), (uint32_t)((q / p.nb) & 1));
    }
    if (p.out == kOutWriteZ) return;

    __syncthreads();
    const int tot = block_compact(nslots, [&](int sl) { return flag[sl] != 0; }, wl, scan_sh);
    for (int i = threadIdx.x; i < tot; i += kStreamThreads) {
        const int sl = wl[i];
        p.lst_idx[c0 + i] = c0 + sl;
        for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + sl) * p.mw + w] = smask[sl * p.mw + w];
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
        float2 a2[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) a2[t] = make_float2(0.f, 0.f);
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
                float2 wf[V / 2];
                unpack2<T>(w[u], wf);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    float2 xf[V / 2];
                    unpack2<T>(xv[u][t], xf);
#pragma unroll
                    for (int e = 0; e < V / 2; ++e) a2[t] = __ffma2_rn(wf[e], xf[e], a2[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(a2[t].x + a2[t].y);
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

bool gate_stream_geometry(int nt, int d, int r, int gate_kind, int cpb, int mw, int* sb, int* nb, size_t* smem) {
    int best_sb = 0, best_nb = 0;
    for (int cand_sb : {8192, 4096, 2048})
        for (int cand_nb = 2; cand_nb <= 4; ++cand_nb) {
            if (gate_stream_smem_bytes(nt, d, r, gate_kind, cpb, mw, cand_sb, cand_nb) > kMaxSmemPerCta) continue;
            const long cur = (long)cand_sb * cand_nb, best = (long)best_sb * best_nb;
            if (cur > best || (cur == best && cand_nb > best_nb)) {
                best_sb = cand_sb;
                best_nb = cand_nb;
            }
        }
    if (!best_sb) return false;
    *sb = best_sb;
    *nb = best_nb;
    *smem = gate_stream_smem_bytes(nt, d, r, gate_kind, cpb, mw, best_sb, best_nb);
    return true;
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
    return launch_ex(kern, dim3(grid), dim3(kStreamThreads), smem, s, pdl, p);
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
