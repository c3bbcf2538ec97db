// Device helpers shared by the gate kernels: fp32 x rows in shared memory,
// 16-byte weight chunks dotted with paired FMAs, and ordered compaction.
#pragma once

#include "common.cuh"

namespace sffn {

// Shared-memory x (and LoPA u) rows are fp32.  For 8-wide (bf16) chunks a row
// of `len` floats holds the first halves of all chunks, then the second
// halves, so consecutive lanes' 16-byte reads hit consecutive banks.
template <int V>
__device__ __forceinline__ int xpos(int len, int c, int e) {
    if (V == 8) return e < 4 ? c * 4 + e : (len >> 1) + c * 4 + (e - 4);
    return c * 4 + e;
}

// A 16-byte weight chunk as element pairs (e0,e1), (e2,e3), ...
template <class WT> __device__ __forceinline__ void unpack2(const uint4& w, float2* f);
template <> __device__ __forceinline__ void unpack2<bf16>(const uint4& w, float2* f) {
    f[0] = make_float2(bf_lo(w.x), bf_hi(w.x));
    f[1] = make_float2(bf_lo(w.y), bf_hi(w.y));
    f[2] = make_float2(bf_lo(w.z), bf_hi(w.z));
    f[3] = make_float2(bf_lo(w.w), bf_hi(w.w));
}
template <> __device__ __forceinline__ void unpack2<float>(const uint4& w, float2* f) {
    f[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
    f[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
}

// acc += <16-byte weight chunk, x chunk c of one token row in shared memory>
// with paired FMAs: acc.x collects the even elements, acc.y the odd ones.
template <class WT>
__device__ __forceinline__ void chunk_dot(const uint4& w, const float* xrow, int len, int c, float2& acc) {
    constexpr int V = Elem<WT>::kVec;
    float2 wf[V / 2];
    unpack2<WT>(w, wf);
    const float4 a = *reinterpret_cast<const float4*>(xrow + xpos<V>(len, c, 0));
    acc = __ffma2_rn(wf[0], make_float2(a.x, a.y), acc);
    acc = __ffma2_rn(wf[1], make_float2(a.z, a.w), acc);
    if (V == 8) {
        const float4 b = *reinterpret_cast<const float4*>(xrow + xpos<V>(len, c, 4));
        acc = __ffma2_rn(wf[2], make_float2(b.x, b.y), acc);
        acc = __ffma2_rn(wf[3], make_float2(b.z, b.w), acc);
    }
}

// Stage tokens [t0, t0 + nt) of a global row-major n x len array (type XT) as
// fp32 rows of `len` in shared memory (chunk layout of weight type WT); rows
// nt..NT-1 are zero.  16-byte loads, all of a thread's loads issued before any
// store (a handful of round trips at most).  All threads of the block take part.
template <class WT, class XT, int NT>
__device__ __forceinline__ void stage_rows(float* dst, const XT* src, int len, int t0, int nt, bool l2_only = false) {
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
            const uint4* q = reinterpret_cast<const uint4*>(src + (size_t)(t0 + t) * len + (size_t)(i - t * per_row) * XV);
            v[u] = (i < total && t < nt) ? (l2_only ? __ldcg(q) : *q) : make_uint4(0u, 0u, 0u, 0u);
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
// L1-bypassing loads (up to 16 in flight per lane); every lane ends with the sums.
template <class WT, int NT>
__device__ __forceinline__ void warp_dot_global(const WT* __restrict__ row, int cpr, const float* xs, int len,
                                                float (&acc)[NT]) {
    constexpr int UB = NT >= 4 ? 8 : 16;
    const int lane = threadIdx.x & 31;
    float2 a2[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) a2[t] = make_float2(0.f, 0.f);
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
                for (int t = 0; t < NT; ++t) chunk_dot<WT>(wv[u], xs + t * len, len, c, a2[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = warp_sum(a2[t].x + a2[t].y);
}

// Per-lane partial of <piece, x_t> over chunks [0, nch) of a shared-memory
// piece whose chunk 0 is chunk `coff` of the row; four chunks' loads are
// issued before their arithmetic.
template <class WT, int NT>
__device__ __forceinline__ void piece_dot(const unsigned char* piece, int nch, int coff, const float* xs, int len,
                                          float2 (&acc)[NT]) {
    const int lane = threadIdx.x & 31;
    const uint4* wp = reinterpret_cast<const uint4*>(piece);
    int c = lane;
    for (; c + 96 < nch; c += 128) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = wp[c + 32 * u];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int t = 0; t < NT; ++t) chunk_dot<WT>(w[u], xs + t * len, len, coff + c + 32 * u, acc[t]);
    }
    for (; c < nch; c += 32) {
        const uint4 w = wp[c];
#pragma unroll
        for (int t = 0; t < NT; ++t) chunk_dot<WT>(w, xs + t * len, len, coff + c, acc[t]);
    }
}

// Per-lane partials of R short rows at once: rows q < cnt of a shared-memory
// piece, rb bytes apart, cpr 16-byte chunks each.  Every lane loads its chunk
// of all R rows before the arithmetic, and the x chunk once for all of them.
template <class WT, int NT, int R>
__device__ __forceinline__ void rows_dot(const unsigned char* piece, int rb, int cnt, int cpr, const float* xs,
                                         int len, float2 (&acc)[R][NT]) {
    const int lane = threadIdx.x & 31;
    for (int c = lane; c < cpr; c += 32) {
        uint4 w[R];
#pragma unroll
        for (int q = 0; q < R; ++q)
            w[q] = q < cnt ? *reinterpret_cast<const uint4*>(piece + (size_t)q * rb + (size_t)c * 16)
                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
            for (int t = 0; t < NT; ++t) chunk_dot<WT>(w[q], xs + t * len, len, c, acc[q][t]);
    }
}

// Warp sums of R values per lane (R = 1, 2, 4 or 8) in log2(R) halving
// exchanges plus 5 - log2(R) plain butterfly steps: the lanes of group
// lane >> (5 - log2 R) end with the sum of v[lane >> (5 - log2 R)].  The
// order of the additions is fixed, so the sums are reproducible.
template <int R>
__device__ __forceinline__ float warp_sum_scatter(const float (&v)[R]) {
    const int lane = threadIdx.x & 31;
    float w[R];
#pragma unroll
    for (int q = 0; q < R; ++q) w[q] = v[q];
    int bit = 16;
#pragma unroll
    for (int m = R; m > 1; m >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < m / 2; ++i) {
            const float send = up ? w[i] : w[i + m / 2];
            const float keep = up ? w[i + m / 2] : w[i];
            w[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    float s = w[0];
    for (; bit > 0; bit >>= 1) s += __shfl_xor_sync(0xffffffffu, s, bit);
    return s;
}

// Ordered compaction of the slots [0, nslots) whose `keep(s)` holds: out[] gets
// them in ascending order; returns the count.  All threads of the block call it.
template <class Keep>
__device__ __forceinline__ int block_compact(int nslots, Keep keep, int* out, int* scan_sh) {
    const int per = (nslots + (int)blockDim.x - 1) / (int)blockDim.x;
    const int sb0 = threadIdx.x * per;
    int cnt = 0;
    for (int q = 0; q < per; ++q)
        if (sb0 + q < nslots && keep(sb0 + q)) ++cnt;
    int tot = 0;
    int pos = block_exclusive_scan(cnt, &tot, scan_sh);
    for (int q = 0; q < per; ++q)
        if (sb0 + q < nslots && keep(sb0 + q)) out[pos++] = sb0 + q;
    __syncthreads();
    return tot;
}

}  // namespace sffn
