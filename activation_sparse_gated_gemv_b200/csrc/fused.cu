// Fused decode path (threshold selection, a few tokens): one kernel streams
// the gate, selects, takes the up dots, and runs the down projection and its
// cross-CTA reduction.
//
// "Model Casting and Low-Parameter Gating" (abstract): the gating matrix is
// evaluated first and the two other matrices are touched only for channels
// whose activation is non-zero.  Here those touches overlap the gate stream:
//
// k_decode, one CTA per SM over its channel range [c0, c0 + cpb), 16 warps
// (LoPA: first each CTA computes its rows of u = x A, and a grid barrier
// publishes u to all CTAs):
//   * warps 0..13 stream the CTA's gate rows (dense W_gate, or LoPA's B) through
//     per-warp rings of bulk copies (TMA engine, mbarriers).  Long rows come in
//     parts whose dot products meet in shared memory; short rows (LoPA's B)
//     come several to a piece and are dotted and selected together.  For a
//     complete row the warp forms z, selects (z > tau) and queues an active
//     channel (with the dense gate and the own-row reduction below, it also
//     pulls the channel's W_up and W_down rows into L2);
//   * with a heavy-hitter set, warps 14 and 15 first take the up dots of the
//     CTA's hot channels, before and independent of the gate;
//   * warps 14 and 15 take queued channels at once and compute the up dot
//     <x, W_up[:,k]> (a hot channel's is already in) and h = (z - tau) u (the
//     streaming warps join them when their pieces are done), so the W_up rows
//     are read while the gate streams;
//   * d <= 4096 (own rows): after a barrier the active channels are compacted
//     in ascending order and every thread adds, for its 8 (or 4) output
//     columns, h_k W_down[k,:] over that ordered list and stores the CTA's
//     fp32 partial of y; a grid-wide barrier (a counter that only grows, so
//     nothing resets it); then every CTA sums one column slice of y over all
//     CTAs' partials in a fixed order and stores it;
//   * larger d (union gather): each CTA publishes its kept-slot mask and h, a
//     grid-wide barrier, then every CTA builds the union's ascending channel
//     list and sums its column slice of h_k W_down[k, slice] over it.
// A host forward with page-locked x passes its device address: the first CTA
// copies x in and the others wait for it on an arrival counter.
// Every sum has a fixed order, so y is bitwise reproducible.
#include "common.cuh"
#include "dot.cuh"

namespace sffn {

constexpr int kDecWarps = 16;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecStreamWarps = 14;        // the other warps start as up workers
constexpr int kQueueTail = 0, kQueueHead = 1, kGateDone = 2, kAbort = 3;

struct DecodeSmem {
    size_t xs, us, zpart, zfin, hs, hu, done, queue, ctr, wl, mask, flag, hrdy, scan, bars, bufs, total;
};

// Chunks (16 bytes of `vec` elements) per column slice of the down pass: the
// smallest power of two covering d with `grid` slices.
__host__ __device__ inline int decode_slice_chunks(int d, int vec, int grid) {
    int cps = 1;
    while (cps * vec * grid < d) cps <<= 1;
    return cps;
}
// Words of a CTA's union mask (one bit per channel slot).
__host__ __device__ inline int decode_mask_words(int cpb) { return (cpb + 31) / 32; }

// The column-slice pass after the grid barrier keeps, in the (then idle)
// streaming ring: every CTA's union mask, the union's ascending channel list
// (at most cpb x grid entries), the per-group partial sums of the slice
// (threads x V x NT floats: kDecThreads / cps groups of NT x cps V) and the
// sub-sums of the fixed-order reduction.
struct DecodeTail {
    size_t masks, list, red, red2, total;
};
__host__ __device__ inline DecodeTail decode_tail_layout(int nt, int cpb, int vec, int grid) {
    DecodeTail T;
    size_t o = 0;
    T.masks = o; o += ((size_t)grid * decode_mask_words(cpb) * 4 + 15) & ~(size_t)15;
    T.list = o;  o += ((size_t)grid * cpb * 4 + 15) & ~(size_t)15;
    T.red = o;   o += (size_t)kDecThreads * vec * nt * sizeof(float);
    T.red2 = o;  o += (size_t)kDecThreads * sizeof(float);
    T.total = o;
    return T;
}
__host__ __device__ inline DecodeSmem decode_smem_layout(int nt, int d, int r, int gate_kind, int cpb, int mw,
                                                         int sb, int nb, int vec, int grid) {
    DecodeSmem L;
    const int glen = gate_kind == kGateLopa ? r : d;
    const int rb = glen * 4;                      // fp32 rows: an upper bound on the part count
    const int ppr = rb <= sb ? 1 : (rb + sb - 1) / sb + 1;
    size_t o = 0;
    L.xs = o;    o += (size_t)nt * d * sizeof(float);
    L.us = o;    o += gate_kind == kGateLopa ? (size_t)nt * r * sizeof(float) : 0;
    L.zpart = o; o += (size_t)cpb * 2 * ppr * nt * sizeof(float);   // x2: dense mode's up parts
    L.zfin = o;  o += (size_t)cpb * nt * sizeof(float);
    L.hs = o;    o += (size_t)cpb * nt * sizeof(float);
    L.hu = o;    o += (size_t)cpb * nt * sizeof(float);
    L.done = o;  o += (size_t)cpb * sizeof(int);
    L.queue = o; o += (size_t)cpb * sizeof(int);
    L.ctr = o;   o += 4 * sizeof(int);
    L.wl = o;    o += (size_t)cpb * sizeof(int);
    L.mask = o;  o += (size_t)cpb * mw * sizeof(uint32_t);
    L.flag = o;  o += ((size_t)cpb + 15) & ~(size_t)15;
    L.hrdy = o;  o += ((size_t)cpb + 15) & ~(size_t)15;
    L.scan = o;  o += 96 * sizeof(int);
    o = (o + 15) & ~(size_t)15;
    L.bars = o;  o += (size_t)kDecStreamWarps * nb * sizeof(uint64_t);
    o = (o + 127) & ~(size_t)127;
    L.bufs = o;
    const size_t ring = (size_t)kDecStreamWarps * nb * sb, tail = decode_tail_layout(nt, cpb, vec, grid).total;
    o += ring > tail ? ring : tail;
    L.total = o;
    return L;
}

// Arrival at a grid barrier on a counter that only grows: the barrier of a
// launch is complete when the counter reaches the next multiple of the grid
// size, so it never needs resetting (64 bits: no wrap in practice).
__device__ __forceinline__ unsigned long long grid_arrive(unsigned long long* ctr, unsigned grid) {
    const unsigned long long old = atomicAdd(ctr, 1ull);
    return (old / grid + 1) * grid;
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

template <class T, int NT, int GATE>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(const DecodeParams p) {
    constexpr int V = Elem<T>::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * p.cpb;
    const int nslots = max(0, min(p.cpb, p.d_ff - c0));
    const int n = p.n;                                  // n <= NT
    const DecodeSmem L = decode_smem_layout(NT, p.d, p.r, GATE, p.cpb, p.mw, p.sb, p.nb, V, gridDim.x);
    const DecodeTail TLd = decode_tail_layout(NT, p.cpb, V, gridDim.x);
    float* xs = reinterpret_cast<float*>(smem + L.xs);
    float* us = reinterpret_cast<float*>(smem + L.us);
    float* zpart = reinterpret_cast<float*>(smem + L.zpart);
    float* zfin = reinterpret_cast<float*>(smem + L.zfin);
    float* hs = reinterpret_cast<float*>(smem + L.hs);
    int* done = reinterpret_cast<int*>(smem + L.done);
    int* queue = reinterpret_cast<int*>(smem + L.queue);
    int* ctr = reinterpret_cast<int*>(smem + L.ctr);
    int* wl = reinterpret_cast<int*>(smem + L.wl);
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + L.mask);
    uint8_t* flag = reinterpret_cast<uint8_t*>(smem + L.flag);
    float* hu = reinterpret_cast<float*>(smem + L.hu);           // hot channels' up dots
    uint8_t* hrdy = reinterpret_cast<uint8_t*>(smem + L.hrdy);   // ... and whether each is in
    int* scan_sh = reinterpret_cast<int*>(smem + L.scan);
    // grid-barrier arrival counters: [0] masks and h published, [1] LoPA's stage 1
    unsigned long long* bar = reinterpret_cast<unsigned long long*>(p.tickets);
    const bool streamer = warp < kDecStreamWarps;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + (streamer ? warp : 0) * p.nb;
    unsigned char* bufs = smem + L.bufs + (size_t)(streamer ? warp : 0) * p.nb * p.sb;

    const int glen = GATE == kGateLopa ? p.r : p.d;
    const float* gx = GATE == kGateLopa ? us : xs;
    const int rb = glen * (int)sizeof(T);
    const int cpr = glen / V;
    const T* wup = static_cast<const T*>(p.wup);
    const T* wdn = static_cast<const T*>(p.wdn);
    const char* gbase = reinterpret_cast<const char*>(static_cast<const T*>(GATE == kGateLopa ? p.bcm : p.wg) +
                                                      (size_t)c0 * glen);
    // Dense FFN mode (dense gate only): every channel is kept, and its W_up row
    // is streamed through the ring right after its gate row, as parts
    // ppr .. 2 ppr - 1 of the channel, so z and the up dot finish together.
    const bool dense = GATE == kGateDense && p.dense;
    const bool rows_mode = !dense && rb <= p.sb;          // pieces of whole rows, else parts of a row
    const char* ubase = reinterpret_cast<const char*>(wup + (size_t)c0 * glen);
    int rpp, ppr, pb;
    if (rows_mode) {
        const int per_warp = (nslots + kDecStreamWarps - 1) / kDecStreamWarps;
        rpp = max(1, min(p.sb / rb, per_warp));
        ppr = 1;
        pb = rpp * rb;
    } else {
        rpp = 1;
        ppr = (rb + p.sb - 1) / p.sb;
        pb = ((rb + ppr - 1) / ppr + 15) & ~15;
        ppr = (rb + pb - 1) / pb;
    }
    const int pps = dense ? 2 * ppr : ppr;               // parts per channel slot
    const int npieces = rows_mode ? (nslots + rpp - 1) / rpp : nslots * pps;
    const int w0 = streamer ? (int)((long long)npieces * warp / kDecStreamWarps) : 0;
    const int wcount = streamer ? (int)((long long)npieces * (warp + 1) / kDecStreamWarps) - w0 : 0;
    const uint64_t pol = l2_evict_first();

    // Cursor over this warp's pieces (w0 + j): row group g, part, ring slot, parity.
    int ig = rows_mode ? w0 : w0 / pps, ipart = rows_mode ? 0 : w0 - (w0 / pps) * pps, ibuf = 0;
    int issued = 0;
    auto issue_next = [&]() {
        uint32_t bytes;
        const char* src;
        if (rows_mode) {
            const int r0 = ig * rpp;
            bytes = (uint32_t)(min(rpp, nslots - r0) * rb);
            src = gbase + (size_t)r0 * rb;
        } else {
            const int q = ipart < ppr ? ipart : ipart - ppr;
            const int off = q * pb;
            bytes = (uint32_t)min(pb, rb - off);
            src = (ipart < ppr ? gbase : ubase) + (size_t)ig * rb + off;
        }
        if (lane == 0) {
            mbar_expect_tx(bars + ibuf, bytes);
            bulk_load(bufs + (size_t)ibuf * p.sb, src, bytes, bars + ibuf, pol);
        }
        if (++ibuf == p.nb) ibuf = 0;
        if (++ipart >= pps) {
            ipart = 0;
            ++ig;
        }
        ++issued;
    };

    if (streamer) {
        if (lane == 0) {
            for (int b = 0; b < p.nb; ++b) mbar_init(bars + b, 1);
            fence_mbar_init();
        }
        __syncwarp();
        // Weights never depend on an earlier kernel: the first piece goes out
        // before the PDL wait, so it lands while the previous kernel finishes;
        // the rest of the ring follows x, which then does not queue behind a
        // full ring of weight traffic.
        while (issued < min(1, wcount)) issue_next();
        __syncwarp();
    }
    // LoPA: this CTA's rows of A^T (stage 1) into L2 as well
    const int u0 = GATE == kGateLopa ? (int)((long long)p.r * blockIdx.x / gridDim.x) : 0;
    const int u1 = GATE == kGateLopa ? (int)((long long)p.r * (blockIdx.x + 1) / gridDim.x) : 0;
    if (GATE == kGateLopa && lane == 0)
        for (int j = u0 + warp; j < u1; j += kDecWarps)
            bulk_prefetch_l2(static_cast<const T*>(p.at) + (size_t)j * p.d, (uint32_t)(p.d * sizeof(T)));

    griddep_wait();
    griddep_launch_dependents();
    // Host buffers: the first xld CTAs pull x from page-locked host memory into
    // the device buffer (16-byte loads, all in flight) and count themselves in
    // on the x counter; every CTA waits for the count before it stages x.
    if (p.xh && (int)blockIdx.x < p.xld) {
        const int n16 = p.n * p.d * (int)sizeof(T) / 16;
        const int per = (n16 + p.xld - 1) / p.xld;
        const int i0 = blockIdx.x * per, i1 = min(n16, i0 + per);
        for (int i = i0 + threadIdx.x; i < i1; i += kDecThreads)
            reinterpret_cast<uint4*>(const_cast<void*>(p.x))[i] = reinterpret_cast<const uint4*>(p.xh)[i];
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(bar + 3, 1ull);
        }
    }

    for (int i = threadIdx.x; i < p.cpb; i += kDecThreads) {
        flag[i] = 0;
        hrdy[i] = 0;
        done[i] = 0;
        queue[i] = 0;
    }
    // Heavy-hitter channels of this CTA, ascending, into the (still unused)
    // list array: one idle warp, ballots.
    if (warp == kDecStreamWarps) {
        int cnt = 0;
        if (p.hot) {
            for (int base = 0; base < nslots; base += 32) {
                const int sl = base + lane;
                const bool hot = sl < nslots && ((__ldg(p.hot + ((c0 + sl) >> 5)) >> ((c0 + sl) & 31)) & 1u);
                const unsigned m = __ballot_sync(0xffffffffu, hot);
                if (hot) wl[cnt + __popc(m & ((1u << lane) - 1u))] = sl;
                cnt += __popc(m);
            }
        }
        if (lane == 0) scan_sh[4] = cnt;
    }
    for (int i = threadIdx.x; i < p.cpb * p.mw; i += kDecThreads) smask[i] = 0u;
    if (threadIdx.x < 4) ctr[threadIdx.x] = 0;
    if (p.xh) {
        if (threadIdx.x == 0) {
            const unsigned long long t0 = globaltimer_ns();
            while (ld_acquire_u64(bar + 3) < p.xtarget) {
                if (globaltimer_ns() - t0 > p.wait_ns) {
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    break;
                }
                __nanosleep(32);
            }
        }
        __syncthreads();
        __threadfence();
    }
    // LoPA stage 1 inside the launch: this CTA's rows of u = x A, published,
    // then a grid barrier, after which every CTA stages all of u.  The rows
    // are dotted with x straight from global memory, so the barrier's arrival
    // does not wait for x's staging (which overlaps the barrier instead); each
    // row is split over `parts` warps, whose sums meet in shared memory (the
    // u staging area, free until then) and are added in part order.  The wait
    // is bounded and cannot deadlock: all CTAs are resident.
    unsigned long long utarget = 0ull;
    if (GATE == kGateLopa) {
        const int nr = u1 - u0;
        const int parts = max(1, min(kDecWarps, p.r) / max(nr, 1));
        float* upart = us;
        const int cpx = p.d / V, per = (cpx + parts - 1) / parts;
        const T* xg = static_cast<const T*>(p.x);
        constexpr int UA = NT <= 1 ? 8 : 4;
        for (int jj = warp; jj < nr * parts; jj += kDecWarps) {
            const int j = u0 + jj / parts, part = jj - (jj / parts) * parts;
            const int ce = min(cpx, (part + 1) * per);
            const T* arow = static_cast<const T*>(p.at) + (size_t)j * p.d;
            float2 a2[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) a2[t] = make_float2(0.f, 0.f);
            for (int cb = part * per + lane; cb < ce; cb += 32 * UA) {
                uint4 wa[UA], xv[UA][NT];
#pragma unroll
                for (int u2 = 0; u2 < UA; ++u2) {
                    const int c = cb + 32 * u2;
                    wa[u2] = c < ce ? ld_stream(arow + (size_t)c * V) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        xv[u2][t] = (c < ce && t < n) ? __ldcg(reinterpret_cast<const uint4*>(xg + (size_t)t * p.d) + c)
                                                      : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u2 = 0; u2 < UA; ++u2) {
                    float2 af[V / 2];
                    unpack2<T>(wa[u2], af);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        float2 xf[V / 2];
                        unpack2<T>(xv[u2][t], xf);
#pragma unroll
                        for (int e = 0; e < V / 2; ++e) a2[t] = __ffma2_rn(af[e], xf[e], a2[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float v = warp_sum(a2[t].x + a2[t].y);
                if (lane == 0) upart[jj * NT + t] = v;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nr * n; i += kDecThreads) {
            const int jr = i / n, t = i - jr * n;
            float sum = 0.f;
            for (int q = 0; q < parts; ++q) sum += upart[(jr * parts + q) * NT + t];
            p.u[(size_t)t * p.r + u0 + jr] = sum;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            utarget = grid_arrive(bar + 1, gridDim.x);
        }
    }
    stage_rows<T, T, NT>(xs, static_cast<const T*>(p.x), p.d, 0, n, p.xh != nullptr);
    if (streamer) {
        while (issued < min(p.nb, wcount)) issue_next();
        __syncwarp();
    }
    __syncthreads();
    if (GATE == kGateLopa) {
        if (threadIdx.x == 0) {
            const unsigned long long target = utarget;
            const unsigned long long t0 = globaltimer_ns();
            unsigned backoff = 32;
            int ok = 1;
            while (ld_acquire_u64(bar + 1) < target) {
                if (globaltimer_ns() - t0 > p.wait_ns) {
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    atomicExch(ctr + kAbort, 1);
                    ok = 0;
                    break;
                }
                __nanosleep(backoff);
                if (backoff < 256) backoff <<= 1;
            }
            scan_sh[3] = ok;
        }
        __syncthreads();
        __threadfence();
        stage_rows<T, float, NT>(us, p.u, p.r, 0, n, true);
        __syncthreads();
    }

    // A selected channel's W_up and W_down rows go to L2 at once when the gate
    // is dense and the CTA sums its own rows (measured: 0.7 us faster on the
    // 7B shape).  With LoPA the prefetches of many channels land in one burst
    // right after the short gate stream (1.7 us slower at 80 % sparsity), and
    // with the union gather the W_down reads are column slices (3.2 us slower).
    const bool l2_prefetch = GATE == kGateDense && p.own_rows;
    // Row s is complete: z from its parts in order, select, queue it.  Dense
    // mode: the up dot is complete too (parts ppr ..), so h is formed here
    // and every channel is kept (with h = 0 for a token whose z <= tau).
    auto finalize = [&](int s) {                         // lane 0 only
        __threadfence_block();
        uint32_t tokmask = 0u;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            float z = 0.f;
            for (int q = 0; q < ppr; ++q) z += zpart[(s * pps + q) * NT + t];
            zfin[s * NT + t] = z;
            if (t < n && z > p.tau) tokmask |= 1u << t;
            if (dense) {
                float u = 0.f;
                for (int q = ppr; q < pps; ++q) u += zpart[(s * pps + q) * NT + t];
                hs[s * NT + t] = (t < n && z > p.tau) ? (z - p.tau) * u : 0.f;
            }
        }
        if (dense) {
            flag[s] = 1;
            smask[s * p.mw] = (1u << n) - 1u;
        } else if (tokmask) {
            flag[s] = 1;
            smask[s * p.mw] = tokmask;                   // n <= 4: tokens sit in mask word 0
            if (l2_prefetch) {
                bulk_prefetch_l2(wdn + (size_t)(c0 + s) * p.d, (uint32_t)(p.d * sizeof(T)));
                bulk_prefetch_l2(wup + (size_t)(c0 + s) * p.d, (uint32_t)(p.d * sizeof(T)));
            }
            const int slot = atomicAdd(ctr + kQueueTail, 1);
            __threadfence_block();
            reinterpret_cast<volatile int*>(queue)[slot] = s + 1;
        }
    };
    // The same for several whole rows at once (pieces of whole rows), each by
    // the lane that has `mine` for it: the lanes select in parallel and take
    // their queue places with one atomic.
    auto finalize_rows = [&](int s, const float (&z)[NT], bool mine) {   // all lanes
        uint32_t tokmask = 0u;
        if (mine) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                zfin[s * NT + t] = z[t];
                if (t < n && z[t] > p.tau) tokmask |= 1u << t;
            }
            if (tokmask) {
                flag[s] = 1;
                smask[s * p.mw] = tokmask;
                if (l2_prefetch) {
                    bulk_prefetch_l2(wdn + (size_t)(c0 + s) * p.d, (uint32_t)(p.d * sizeof(T)));
                    bulk_prefetch_l2(wup + (size_t)(c0 + s) * p.d, (uint32_t)(p.d * sizeof(T)));
                }
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, tokmask != 0u);
        if (m) {
            int base = 0;
            if (lane == 0) base = atomicAdd(ctr + kQueueTail, __popc(m));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (tokmask) {
                __threadfence_block();
                reinterpret_cast<volatile int*>(queue)[base + __popc(m & ((1u << lane) - 1u))] = s + 1;
            }
        }
    };

    // ---- streaming warps
    if (streamer) {
        int cbuf = 0, cpar = 0;
        int g = rows_mode ? w0 : w0 / pps, part = rows_mode ? 0 : w0 - (w0 / pps) * pps;
        bool abort = false;
        int abort_at = 0;
        for (int j = 0; j < wcount; ++j) {
            if (!abort && !mbar_wait_warp(bars + cbuf, (uint32_t)cpar)) {
                abort = true;
                abort_at = j;
                if (lane == 0) {
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    atomicExch(ctr + kAbort, 1);
                }
            }
            if (!abort) {
                const unsigned char* buf = bufs + (size_t)cbuf * p.sb;
                if (rows_mode) {
                    // R rows at a time: the dots, one scattering warp sum
                    // that leaves row q's z with lane group q, and the
                    // selection by the first lane of each group
                    constexpr int R = NT <= 2 ? 8 : 4;
                    constexpr int GS = 32 / R;                   // lanes per row group
                    const int r0 = g * rpp, cnt = min(rpp, nslots - r0);
                    for (int q0 = 0; q0 < cnt; q0 += R) {
                        float2 v2[R][NT];
#pragma unroll
                        for (int q = 0; q < R; ++q)
#pragma unroll
                            for (int t = 0; t < NT; ++t) v2[q][t] = make_float2(0.f, 0.f);
                        rows_dot<T, NT, R>(buf + (size_t)q0 * rb, rb, min(R, cnt - q0), cpr, gx, glen, v2);
                        float z[NT];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            float v[R];
#pragma unroll
                            for (int q = 0; q < R; ++q) v[q] = v2[q][t].x + v2[q][t].y;
                            z[t] = warp_sum_scatter<R>(v);
                        }
                        const int q = lane / GS;
                        finalize_rows(r0 + q0 + q, z, lane % GS == 0 && q0 + q < cnt);
                    }
                } else {
                    const int off = (part < ppr ? part : part - ppr) * pb;
                    float2 v2[NT];
#pragma unroll
                    for (int t = 0; t < NT; ++t) v2[t] = make_float2(0.f, 0.f);
                    piece_dot<T, NT>(buf, min(pb, rb - off) >> 4, off >> 4, gx, glen, v2);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float v = warp_sum(v2[t].x + v2[t].y);
                        if (lane == t) zpart[(g * pps + part) * NT + t] = v;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        __threadfence_block();
                        if (atomicAdd(done + g, 1) == pps - 1) finalize(g);
                    }
                }
                __syncwarp();
                if (issued < wcount) {
                    if (lane == 0) fence_proxy_async();
                    issue_next();
                }
            }
            if (++cbuf == p.nb) {
                cbuf = 0;
                cpar ^= 1;
            }
            if (++part >= pps) {
                part = 0;
                ++g;
            }
        }
        if (abort) {
            for (int q = abort_at; q < issued; ++q)
                mbar_wait_warp(bars + (q % p.nb), (uint32_t)((q / p.nb) & 1));
        }
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            atomicAdd(ctr + kGateDone, 1);
        }
    }

    // ---- heavy hitters: the two warps that are not streaming take the up dots
    // of the CTA's hot channels at once, independent of the gate (each is
    // used if the gate selects its channel)
    if (!streamer) {
        const int nhot = scan_sh[4];
        for (int j = warp - kDecStreamWarps; j < nhot; j += kDecWarps - kDecStreamWarps) {
            const int sl = wl[j];
            float u[NT];
            warp_dot_global<T, NT>(wup + (size_t)(c0 + sl) * p.d, p.d / V, xs, p.d, u);
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (lane == t) hu[sl * NT + t] = u[t];
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                reinterpret_cast<volatile uint8_t*>(hrdy)[sl] = 1;
            }
        }
    }

    // ---- up workers (all warps once their streaming is done)
    for (;;) {
        int i = 0;
        if (lane == 0) i = atomicAdd(ctr + kQueueHead, 1);
        i = __shfl_sync(0xffffffffu, i, 0);
        if (i >= nslots) break;
        int s = 0;
        if (lane == 0) {
            const unsigned long long t0 = globaltimer_ns();
            for (;;) {
                s = reinterpret_cast<volatile int*>(queue)[i];
                if (s) break;
                const volatile int* vc = ctr;
                if ((vc[kGateDone] == kDecStreamWarps && vc[kQueueTail] <= i) || vc[kAbort]) break;
                __nanosleep(64);
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    atomicExch(ctr + kAbort, 1);
                    break;
                }
            }
            __threadfence_block();
        }
        s = __shfl_sync(0xffffffffu, s, 0);
        if (!s) break;
        --s;
        __syncwarp();
        const int k = c0 + s;
        float u[NT];
        int ready = 0;
        if (lane == 0) ready = reinterpret_cast<volatile uint8_t*>(hrdy)[s];
        if (__shfl_sync(0xffffffffu, ready, 0)) {
            // a heavy hitter whose up dot is in (the same dot, so the same h)
            __threadfence_block();
#pragma unroll
            for (int t = 0; t < NT; ++t) u[t] = hu[s * NT + t];
        } else {
            warp_dot_global<T, NT>(wup + (size_t)k * p.d, p.d / V, xs, p.d, u);
        }
        const uint32_t tokmask = smask[s * p.mw];
#pragma unroll
        for (int t = 0; t < NT; ++t)
            if (lane == t && t < n) {
                const float h = ((tokmask >> t) & 1u) ? (zfin[s * NT + t] - p.tau) * u[t] : 0.f;
                hs[s * NT + t] = h;
            }
    }
    __syncthreads();

    if (dense || p.own_rows) {
        // ---- own rows: the CTA's kept slots in ascending order (every slot in
        // the dense FFN).  Each thread adds, for its 16-byte column chunks,
        // h_k W_down[k, :] over those rows (16 rows in flight), stores the CTA's
        // fp32 partial of y, and after a grid barrier every CTA sums one column
        // slice of y over the partials in CTA order.
        int tot = nslots;
        if (!dense) {
            if (warp == 0) {
                int cnt = 0;
                for (int base = 0; base < nslots; base += 32) {
                    const int sl = base + lane;
                    const bool f = sl < nslots && flag[sl];
                    const unsigned m = __ballot_sync(0xffffffffu, f);
                    if (f) wl[cnt + __popc(m & ((1u << lane) - 1u))] = sl;
                    cnt += __popc(m);
                }
                if (lane == 0) scan_sh[0] = cnt;
            }
            __syncthreads();
            tot = scan_sh[0];
        }
        auto slot_of = [&](int i) { return dense ? i : wl[i]; };
        constexpr int UBD = 16;
        const int cpd = p.d / V;                          // 16-byte chunks per output row
        for (int cch = threadIdx.x; cch < cpd; cch += kDecThreads) {
            float2 acc[NT][V / 2];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < V / 2; ++e) acc[t][e] = make_float2(0.f, 0.f);
            for (int s0 = 0; s0 < tot; s0 += UBD) {
                uint4 w[UBD];
#pragma unroll
                for (int u2 = 0; u2 < UBD; ++u2) {
                    if (s0 + u2 >= tot) {
                        w[u2] = make_uint4(0u, 0u, 0u, 0u);
                    } else {
                        const T* src = wdn + (size_t)(c0 + slot_of(s0 + u2)) * p.d + (size_t)cch * V;
                        w[u2] = dense ? ld_stream_nc(src) : ld_stream(src);
                    }
                }
#pragma unroll
                for (int u2 = 0; u2 < UBD; ++u2) {
                    if (s0 + u2 < tot) {
                        float wf[V];
                        unpack<T>(w[u2], wf);
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            const float h = hs[slot_of(s0 + u2) * NT + t];
                            const float2 hh = make_float2(h, h);
#pragma unroll
                            for (int e = 0; e < V / 2; ++e)
                                acc[t][e] = __ffma2_rn(make_float2(wf[2 * e], wf[2 * e + 1]), hh, acc[t][e]);
                        }
                    }
                }
            }
            for (int t = 0; t < n; ++t) {
                float* dst = p.part + ((size_t)blockIdx.x * n + t) * p.d + (size_t)cch * V;
#pragma unroll
                for (int e = 0; e < V / 2; e += 2)
                    *reinterpret_cast<float4*>(dst + 2 * e) =
                        make_float4(acc[t][e].x, acc[t][e].y, acc[t][e + 1].x, acc[t][e + 1].y);
            }
        }
        const int G = gridDim.x;
        const int cps = decode_slice_chunks(p.d, V, G);
        const int col0 = blockIdx.x * cps * V;
        __syncthreads();
        unsigned long long target = 0ull;
        if (threadIdx.x == 0) {
            __threadfence();                              // release: the CTA's partial first
            if (col0 < p.d) target = grid_arrive(bar, G) + (unsigned long long)p.bar_extra;
            else atomicAdd(bar, 1ull);
        }
        // the CTA's list, for sffn_get_active only: off the path to the barrier
        for (int i = threadIdx.x; i < tot; i += kDecThreads) {
            const int sl = slot_of(i);
            p.lst_idx[c0 + i] = c0 + sl;
            for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + sl) * p.mw + w] = smask[sl * p.mw + w];
        }
        if (threadIdx.x == 0) {
            p.seg_count[blockIdx.x] = tot;
            int ok = 1;
            if (col0 < p.d) {
                const unsigned long long t0 = globaltimer_ns();
                unsigned backoff = 32;
                while (ld_acquire_u64(bar) < target) {
                    if (globaltimer_ns() - t0 > p.wait_ns) {
                        raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                        ok = 0;
                        break;
                    }
                    __nanosleep(backoff);
                    if (backoff < 256) backoff <<= 1;
                }
            }
            scan_sh[2] = ok;
        }
        __syncthreads();
        if (!scan_sh[2] || col0 >= p.d) return;
        __threadfence();
        // y[:, col0 : col0 + cps V] = sum over the G partials: thread (g, item)
        // adds partials g, g + GR, ... in order (up to UBS loads in flight),
        // then the GR sums in order; GR is as small as one round of loads
        // allows, so that the serial second sum is short
        constexpr int UBS = 16;
        const int q4 = min(cps * V, p.d - col0) / 4;      // float4 per token
        const int items = n * q4;
        const int GR = max(1, min(kDecThreads / items, (G + UBS - 1) / UBS));
        float4* red4 = reinterpret_cast<float4*>(smem + L.bufs);          // the idle ring
        const int g = (int)threadIdx.x / items, item = (int)threadIdx.x - g * items;
        if (g < GR) {
            const int t = item / q4, c = col0 + (item - t * q4) * 4;
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int b0 = g; b0 < G; b0 += UBS * GR) {
                float4 v[UBS];
#pragma unroll
                for (int u2 = 0; u2 < UBS; ++u2) {
                    const int b = b0 + u2 * GR;
                    v[u2] = b < G ? __ldcg(reinterpret_cast<const float4*>(p.part + ((size_t)b * n + t) * p.d + c))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u2 = 0; u2 < UBS; ++u2)
                    if (b0 + u2 * GR < G) {
                        sum.x += v[u2].x; sum.y += v[u2].y; sum.z += v[u2].z; sum.w += v[u2].w;
                    }
            }
            red4[g * items + item] = sum;
        }
        __syncthreads();
        if ((int)threadIdx.x < items) {
            float4 sum = red4[threadIdx.x];
            for (int q = 1; q < GR; ++q) {
                const float4 v = red4[q * items + threadIdx.x];
                sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
            }
            const int t = (int)threadIdx.x / q4, c = col0 + ((int)threadIdx.x - t * q4) * 4;
            T* dst = static_cast<T*>(p.y) + (size_t)t * p.d + c;
            dst[0] = from_f32<T>(sum.x);
            dst[1] = from_f32<T>(sum.y);
            dst[2] = from_f32<T>(sum.z);
            dst[3] = from_f32<T>(sum.w);
        }
        return;
    }

    // ---- publish this CTA's part of the union: one mask bit per slot that
    // some token selected, and h for those slots (every token; 0 for a token
    // that did not select the channel)
    const int mwc = decode_mask_words(p.cpb);
    for (int w = threadIdx.x; w < mwc; w += kDecThreads) {
        uint32_t m = 0u;
        for (int i = 0; i < 32; ++i) {
            const int sl = 32 * w + i;
            if (sl < nslots && flag[sl]) m |= 1u << i;
        }
        p.umask[(size_t)blockIdx.x * mwc + w] = m;
    }
    for (int i = threadIdx.x; i < nslots * n; i += kDecThreads) {
        const int sl = i / n, t = i - sl * n;
        if (flag[sl]) p.lst_h[(size_t)(c0 + sl) * n + t] = hs[sl * NT + t];
    }

    // ---- grid barrier: every CTA's mask and h are out.  All CTAs are
    // resident (a cooperative launch of one CTA per SM), so the wait ends; it
    // is bounded all the same.  A CTA without a column slice of y only arrives.
    const int G = gridDim.x;
    const int cps = decode_slice_chunks(p.d, V, G);       // 16-byte chunks per column slice
    const int col0 = blockIdx.x * cps * V;
    __syncthreads();
    unsigned long long target = 0ull;
    if (threadIdx.x == 0) {
        __threadfence();                                  // release: the CTA's mask and h first
        if (col0 < p.d) target = grid_arrive(bar, G) + (unsigned long long)p.bar_extra;
        else atomicAdd(bar, 1ull);
    }
    // the CTA's ascending list and token masks, for sffn_get_active only: off
    // the path to the barrier (one warp, ballots)
    if (warp == 0) {
        int cnt = 0;
        for (int base = 0; base < nslots; base += 32) {
            const int sl = base + lane;
            const bool f = sl < nslots && flag[sl];
            const unsigned m = __ballot_sync(0xffffffffu, f);
            if (f) {
                const int i = cnt + __popc(m & ((1u << lane) - 1u));
                p.lst_idx[c0 + i] = c0 + sl;
                for (int w = 0; w < p.mw; ++w) p.lst_mask[(size_t)(c0 + sl) * p.mw + w] = smask[sl * p.mw + w];
            }
            cnt += __popc(m);
        }
        if (lane == 0) p.seg_count[blockIdx.x] = cnt;
    }
    if (threadIdx.x == 0) {
        int ok = 1;
        if (col0 < p.d) {
            const unsigned long long t0 = globaltimer_ns();
            unsigned backoff = 32;
            while (ld_acquire_u64(bar) < target) {
                if (globaltimer_ns() - t0 > p.wait_ns) {
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    ok = 0;
                    break;
                }
                __nanosleep(backoff);
                if (backoff < 256) backoff <<= 1;
            }
        }
        scan_sh[2] = ok;
    }
    __syncthreads();
    if (!scan_sh[2] || col0 >= p.d) return;
    __threadfence();

    // ---- y[:, col0 : col0 + cps V] = sum over the union, in ascending channel
    // order, of h[k] W_down[k, slice].  The W_down rows were pulled into L2
    // when their channels were selected, so the slices come from L2.
    uint32_t* gm = reinterpret_cast<uint32_t*>(smem + L.bufs + TLd.masks);     // [G][mwc]
    int* list = reinterpret_cast<int*>(smem + L.bufs + TLd.list);             // [<= G cpb], ascending
    float* red = reinterpret_cast<float*>(smem + L.bufs + TLd.red);            // [groups][NT][slice]
    float* red2 = reinterpret_cast<float*>(smem + L.bufs + TLd.red2);          // [kDecThreads]
    // every CTA's union mask, all loads in flight before any store
    const int nw = G * mwc;
    {
        constexpr int UM = 4;
        uint32_t v[UM];
#pragma unroll
        for (int u = 0; u < UM; ++u) {
            const int i = (int)threadIdx.x + u * kDecThreads;
            v[u] = i < nw ? __ldcg(p.umask + i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < UM; ++u) {
            const int i = (int)threadIdx.x + u * kDecThreads;
            if (i < nw) gm[i] = v[u];
        }
        for (int i = (int)threadIdx.x + UM * kDecThreads; i < nw; i += kDecThreads) gm[i] = __ldcg(p.umask + i);
    }
    __syncthreads();
    // the union's channels in ascending order: word i is CTA i / mwc's slots
    // 32 (i % mwc) .. + 31, so word order is channel order
    const int per = (nw + kDecThreads - 1) / kDecThreads;
    const int wa = min(nw, (int)threadIdx.x * per), wb = min(nw, wa + per);
    int cw = 0;
    for (int i = wa; i < wb; ++i) cw += __popc(gm[i]);
    int U = 0;
    int pos = block_exclusive_scan(cw, &U, scan_sh + 48);
    for (int i = wa; i < wb; ++i) {
        uint32_t m = gm[i];
        const int b = i / mwc, base = b * p.cpb + 32 * (i - b * mwc);
        while (m) {
            list[pos++] = base + __ffs(m) - 1;
            m &= m - 1u;
        }
    }
    __syncthreads();

    // thread (group g, chunk cc): rows g, g + NG, ... of the list, 16 bytes each
    const int NG = kDecThreads / cps;
    const int g = (int)threadIdx.x / cps, cc = (int)threadIdx.x - g * cps;
    const int col = col0 + cc * V;
    const bool colok = col < p.d;
    float2 acc[NT][V / 2];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < V / 2; ++e) acc[t][e] = make_float2(0.f, 0.f);
    constexpr int UB = NT == 1 ? 16 : 8;                  // a group's rows in flight: usually all of them
    for (int i0 = g; i0 < U; i0 += UB * NG) {
        uint4 w[UB];
        float hv[UB][NT];
#pragma unroll
        for (int u2 = 0; u2 < UB; ++u2) {
            const int i = i0 + u2 * NG;
            const int k = i < U ? list[i] : -1;
            w[u2] = (k >= 0 && colok) ? ld_stream(wdn + (size_t)k * p.d + col) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int t = 0; t < NT; ++t) hv[u2][t] = (k >= 0 && t < n) ? __ldcg(p.lst_h + (size_t)k * n + t) : 0.f;
        }
#pragma unroll
        for (int u2 = 0; u2 < UB; ++u2) {
            float wf[V];
            unpack<T>(w[u2], wf);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const float2 hh = make_float2(hv[u2][t], hv[u2][t]);
#pragma unroll
                for (int e = 0; e < V / 2; ++e)
                    acc[t][e] = __ffma2_rn(make_float2(wf[2 * e], wf[2 * e + 1]), hh, acc[t][e]);
            }
        }
    }
    // fixed-order sum over the NG groups: Q sub-sums of consecutive groups,
    // then the Q sub-sums in order
    const int SC = cps * V;
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < V / 2; ++e)
            *reinterpret_cast<float2*>(red + ((size_t)g * NT + t) * SC + cc * V + 2 * e) = acc[t][e];
    __syncthreads();
    const int items = n * SC;
    const int Q = kDecThreads / items;                    // >= 1 (the geometry checks n SC <= threads)
    const int GPQ = (NG + Q - 1) / Q;
    {
        const int q = (int)threadIdx.x / items, it = (int)threadIdx.x - q * items;
        if (q < Q) {
            const int t = it / SC, j = it - t * SC;
            float sum = 0.f;
            const int ga = q * GPQ, gb = min(NG, ga + GPQ);
            for (int gg = ga; gg < gb; ++gg) sum += red[((size_t)gg * NT + t) * SC + j];
            red2[q * items + it] = sum;
        }
    }
    __syncthreads();
    if ((int)threadIdx.x < items) {
        const int it = threadIdx.x, t = it / SC, j = it - t * SC;
        float sum = 0.f;
        for (int q = 0; q < Q; ++q) sum += red2[q * items + it];
        if (col0 + j < p.d) static_cast<T*>(p.y)[(size_t)t * p.d + col0 + j] = from_f32<T>(sum);
    }
}

// ---------------------------------------------------------------------------

size_t decode_smem_bytes(int nt, int d, int r, int gate_kind, int cpb, int mw, int sb, int nb, int vec, int grid) {
    return decode_smem_layout(nt, d, r, gate_kind, cpb, mw, sb, nb, vec, grid).total;
}

bool decode_geometry(int nt, int d, int r, int gate_kind, int cpb, int mw, int vec, int grid, int* sb, int* nb,
                     size_t* smem) {
    // the column-slice pass gives one thread to each (token, column) of a slice
    // in its last step, and at least one thread to each 16-byte chunk
    const int cps = grid < 1 ? 0 : decode_slice_chunks(d, vec, grid);
    if (grid < 1 || (long)nt * cps * vec > kDecThreads || cps > kDecThreads) return false;
    int best_sb = 0, best_nb = 0;
    for (int cand_sb : {8192, 4096, 2048})
        for (int cand_nb = 2; cand_nb <= 4; ++cand_nb) {
            if (decode_smem_bytes(nt, d, r, gate_kind, cpb, mw, cand_sb, cand_nb, vec, grid) > kMaxSmemPerCta)
                continue;
            const long cur = (long)cand_sb * cand_nb, best = (long)best_sb * best_nb;
            if (cur > best || (cur == best && cand_nb > best_nb)) {
                best_sb = cand_sb;
                best_nb = cand_nb;
            }
        }
    if (!best_sb) return false;
    *sb = best_sb;
    *nb = best_nb;
    *smem = decode_smem_bytes(nt, d, r, gate_kind, cpb, mw, best_sb, best_nb, vec, grid);
    return true;
}

template <class T, int NT, int GATE>
static cudaError_t launch_decode_t(const DecodeParams& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
    auto kern = k_decode<T, NT, GATE>;
    static SmemAttrCache cache;
    cudaError_t e = ensure_smem(kern, smem, cache);
    if (e != cudaSuccess) return e;
    // cooperative: the kernel's grid barriers need every CTA resident at once
    return launch_ex(kern, dim3(grid), dim3(kDecThreads), smem, s, pdl, p, true);
}

template <class T, int NT>
static cudaError_t launch_decode_nt(const DecodeParams& p, int gate_kind, int grid, size_t smem, cudaStream_t s,
                                    bool pdl) {
    return gate_kind == kGateLopa ? launch_decode_t<T, NT, kGateLopa>(p, grid, smem, s, pdl)
                                  : launch_decode_t<T, NT, kGateDense>(p, grid, smem, s, pdl);
}

cudaError_t launch_decode(int wdtype, const DecodeParams& p, int nt, int gate_kind, int grid, size_t smem,
                          cudaStream_t s, bool pdl) {
    if (p.n > nt || p.mw < 1 || p.sb <= 0 || p.sb % 16 || p.nb <= 0) return cudaErrorInvalidValue;
    if (wdtype == 0) {
        switch (nt) {
            case 1: return launch_decode_nt<bf16, 1>(p, gate_kind, grid, smem, s, pdl);
            case 2: return launch_decode_nt<bf16, 2>(p, gate_kind, grid, smem, s, pdl);
            case 4: return launch_decode_nt<bf16, 4>(p, gate_kind, grid, smem, s, pdl);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (nt) {
        case 1: return launch_decode_nt<float, 1>(p, gate_kind, grid, smem, s, pdl);
        case 2: return launch_decode_nt<float, 2>(p, gate_kind, grid, smem, s, pdl);
        case 4: return launch_decode_nt<float, 4>(p, gate_kind, grid, smem, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sffn
