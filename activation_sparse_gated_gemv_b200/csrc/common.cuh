// Shared device helpers and launch-parameter structs for the sffn kernels.
//
// Data layout in HBM (all channel-major so an active channel is one row):
//   wg   [d_ff][d]   gate column k of W_gate as row k        (dense gate)
//   a    [d][r]      LoPA first factor, row-major as given
//   bcm  [d_ff][r]   LoPA second factor, column k of B as row k
//   wup  [d_ff][d]   column k of W_up as row k
//   wdn  [d_ff][d]   W_down as given (row k is channel k)
// Workspace (library-owned):
//   zbuf [n][d_ff] f32   gate values, written only when a later kernel needs them (top-K)
//   gbuf [n][d_ff] f32   top-K activation SiLU(z) on selected channels, 0 elsewhere
//   sel  [n][d_ff] u8    top-K selection flags
//   lst_idx [d_ff]       per-CTA segments of ascending active channel ids
//   lst_h   [d_ff][n]    h[k][t] = g[t,k] <x_t, W_up[:,k]>, valid for listed k
//   lst_mask[d_ff][mw]   bit t of channel k: token t selected k
//   seg_count[g1]        entries in each gate CTA's segment
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sffn {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTokens = 1024;

using bf16 = __nv_bfloat16;

template <class T> struct Elem;
template <> struct Elem<bf16> { static constexpr int kVec = 8; };
template <> struct Elem<float> { static constexpr int kVec = 4; };

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start before its predecessor ends; it must wait here before
// touching anything the predecessor (or an earlier kernel) reads or writes.
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte streaming load of read-only weights: bypasses L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// bf16 is the upper half of an IEEE binary32: widening is a 16-bit shift.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// A 16-byte chunk as floats.
template <class T> __device__ __forceinline__ void unpack(const uint4& v, float* f);
template <> __device__ __forceinline__ void unpack<bf16>(const uint4& v, float* f) {
    f[0] = bf_lo(v.x); f[1] = bf_hi(v.x);
    f[2] = bf_lo(v.y); f[3] = bf_hi(v.y);
    f[4] = bf_lo(v.z); f[5] = bf_hi(v.z);
    f[6] = bf_lo(v.w); f[7] = bf_hi(v.w);
}
template <> __device__ __forceinline__ void unpack<float>(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

template <class T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }

template <class T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exclusive prefix sum of one int per thread over the block, in thread order.
// `sh` holds at least 33 ints.  Every thread of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? sh[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sh[lane] = w;
    }
    __syncthreads();
    const int before = warp ? sh[warp - 1] : 0;
    *total = sh[nwarps - 1];
    __syncthreads();
    return before + x - v;
}

// ---------------------------------------------------------------------------
// Launch parameters.

enum GateKind { kGateDense = 0, kGateLopa = 1, kGatePreselected = 2 };
enum GateOut { kOutSelectUp = 0, kOutWriteZ = 1 };

struct GateParams {
    const void* x;          // [n][d] T
    int n, d, d_ff, r;
    const void* wg;         // [d_ff][d]      dense gate rows
    const void* bcm;        // [d_ff][r]      LoPA B rows
    const float* u;         // [n][r]         LoPA x A
    const void* wup;        // [d_ff][d]
    int out;                // GateOut
    int force_all;          // dense FFN: every channel is listed
    float tau;              // threshold
    float* zbuf;            // [n][d_ff] (kOutWriteZ)
    const float* gbuf;      // [n][d_ff] (kGatePreselected)
    const uint8_t* sel;     // [n][d_ff] (kGatePreselected)
    int cpb;                // channels per CTA
    int mw;                 // mask words per channel
    int* lst_idx;
    float* lst_h;
    uint32_t* lst_mask;
    int* seg_count;
};

struct LopaUParams {
    const void* x;          // [n][d] T
    const void* a;          // [d][r] T
    int n, d, r;
    int rows_per_cta;       // d split
    int cols_per_cta;       // r split (multiple of the vector width)
    float* part;            // [splits][n][r]
    float* u;               // [n][r]
    unsigned* tickets;      // [r column groups]
};

struct TopkParams {
    const float* zbuf;      // [n][d_ff]
    int n, d_ff, k;
    float* gbuf;            // [n][d_ff]
    uint8_t* sel;           // [n][d_ff]
};

struct DownParams {
    const void* wdn;        // [d_ff][d] T
    int n, d, d_ff;
    const int* seg_count;   // [g1]
    int g1, cpb;
    const int* lst_idx;
    const float* lst_h;     // [d_ff][n]
    float* part;            // [chunks][n][d]
    unsigned* tickets;      // [column slices]
    void* y;                // [n][d] T
    int chunks;             // chunk CTAs per column slice (grid.y)
    int min_rows;           // fewest rows worth a chunk
    int max_rows;           // rows one chunk can hold (shared-memory bound)
    int* status;            // sticky device status word (bit set on a failed check)
};

// Bits of the device status word.
enum StatusBits { kStatusDownRows = 1 };

// Raise a kernel's dynamic shared-memory limit once per device (so a forward
// inside stream capture issues launches only).  `cache` is per kernel.
struct SmemAttrCache {
    int bytes[64] = {};
};
template <class K>
inline cudaError_t ensure_smem(K kernel, size_t smem, SmemAttrCache& cache) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((int)smem <= cache.bytes[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) cache.bytes[dev] = (int)smem;
    return e;
}

// Launch with programmatic dependent launch (PDL) when `pdl` is set.
template <class K, class P>
inline cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             const P& params) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, params);
}

// Host-side launchers (one per kernel family); return cudaError_t.
cudaError_t launch_gate(int wdtype, const GateParams& p, int nt, int rw, int gate_kind, int grid,
                        size_t smem, cudaStream_t s, bool pdl);
size_t gate_smem_bytes(int wdtype, int nt, int d, int r, int gate_kind, int cpb, int mw);
cudaError_t launch_lopa_u(int wdtype, const LopaUParams& p, int nt, dim3 grid, cudaStream_t s,
                          bool pdl);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_down(int wdtype, const DownParams& p, int nt, int slices, size_t smem,
                        cudaStream_t s, bool pdl);
size_t down_smem_bytes(int wdtype, int nt, int g1, int max_rows);
int down_max_rows(int d_ff, int chunks, int min_rows);
int down_slice_cols(int wdtype);
cudaError_t launch_transpose(int wdtype, const void* src, void* dst, int rows, int cols,
                             cudaStream_t s);

}  // namespace sffn
