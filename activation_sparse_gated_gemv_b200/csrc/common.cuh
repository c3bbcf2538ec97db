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
#include <cuda.h>
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

// 16-byte load of weights read once, cached in L2 only.  (The non-coherent
// path, ld.global.nc, measured much slower for these row reads behind a full
// stream of bulk copies: an 8 KB up-dot row took 3.7-4.5 us instead of
// 2.1-2.6 us at the end of the gate stream.)
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}
// The same through the non-coherent path without L1 allocation: faster for
// the dense FFN's sweep of every W_down row (53.8 against 52.7 us on the 7B
// shape).
__device__ __forceinline__ uint4 ld_stream_nc(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Bulk asynchronous copies (TMA engine, 1-D form) completing on an mbarrier.
// No cluster multicast anywhere: every copy lands in the issuing CTA.

constexpr unsigned long long kWaitLimitNs = 500ull * 1000ull * 1000ull;   // 0.5 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Orders this thread's generic-proxy global accesses with its async-proxy ones
// (bulk copies).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
// Global -> this CTA's shared memory, `bytes` a multiple of 16, both ends 16-byte aligned.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
// Ask the TMA engine to bring `bytes` (multiple of 16) at `src` into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// L2 policy for data read once per forward (weights): evict first.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// Waits (suspended, up to a hint of about 1 ms) for the phase with `parity`
// to complete; false if it has not completed by then.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Every lane of the warp waits for the phase with `parity` to complete.  The
// decision is warp-uniform; false after kWaitLimitNs (the caller records it).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
    bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (!done) done = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        const bool late = globaltimer_ns() - t0 > kWaitLimitNs;
        if (__shfl_sync(0xffffffffu, late ? 1 : 0, 0)) return false;
    }
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
    const void* wdn;        // [d_ff][d]      W_down rows (L2 prefetch of active channels), may be NULL
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
    int sb;                 // streamed piece bytes (multiple of 16)
    int nb;                 // pieces in flight per warp
    int* status;            // sticky device status word
    int* hstatus;           // its host-mapped mirror, or NULL
};

struct LopaUParams {
    const void* x;          // [n][d] T
    const void* at;         // [r][d] T   A transposed: column j of A is row j
    int n, d, r;
    float* u;               // [n][r]
};

struct TopkParams {
    const float* zbuf;      // [n][d_ff]
    int n, d_ff, k;
    float* gbuf;            // [n][d_ff]
    uint8_t* sel;           // [n][d_ff]
    uint32_t* ubits;        // [d_ff/32] union bitmap, OR-ed into (NULL: none)
    int mode;               // 0: top-K (k channels), 1: top-p (softmax mass p)
    float p;
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
    int chunks;             // chunk CTAs per column slice (grid.y), each a run of gate segments
    int* status;            // sticky device status word (bit set on a failed check)
    int* hstatus;           // its host-mapped mirror, or NULL
};

struct DecodeParams {
    const void* x;          // [n][d] T, n <= the token tile
    int n, d, d_ff, r;
    const void* wg;         // [d_ff][d]   dense gate rows
    const void* bcm;        // [d_ff][r]   LoPA B rows
    const void* at;         // [r][d]      LoPA A^T rows (stage 1 inside the kernel)
    float* u;               // [n][r]      LoPA x A, written and read inside the kernel
    const void* wup;        // [d_ff][d]
    const void* wdn;        // [d_ff][d]
    float tau;
    int cpb, mw;
    int* lst_idx;           // [CTAs][cpb] each CTA's active channels, ascending (for sffn_get_active)
    float* lst_h;           // [d_ff][n] h of the union's channels (0 for a token that did not select one)
    uint32_t* lst_mask;     // [d_ff][mw] (for sffn_get_active)
    int* seg_count;         // [CTAs] (for sffn_get_active)
    uint32_t* umask;        // [CTAs][ceil(cpb / 32)] union mask of each CTA's channel slots
    float* part;            // dense mode: [CTAs][n][d] per-CTA partials of y
    int sb, nb;             // streamed piece bytes, pieces in flight per streaming warp
    int* status;
    int* hstatus;           // host-mapped mirror of the status word, or NULL
    unsigned long long wait_ns;   // limit of the grid-barrier waits
    int bar_extra;          // arrivals the final grid barrier expects beyond the grid (0; 1 makes it time out)
    unsigned* tickets;      // 64-bit arrival counters (h, LoPA's u, the union masks, x), zero at creation
    void* y;                // [n][d] T
    const uint32_t* hot;    // [ceil(d_ff / 32)] heavy-hitter channel bits, or NULL
    int dense;              // dense FFN (dense gate): every channel, W_up rows streamed with the gate's
    int own_rows;           // sparse: reduce through per-CTA partials of y instead of the union gather
    const void* xh;         // forward with host buffers: device address of the page-locked host copy of x,
                            // pulled into x (device memory) inside the launch; NULL when x is already there
    int xld;                // CTAs that pull x (the first xld)
    unsigned long long xtarget;   // arrivals the x counter (tickets' fourth word) reaches once x is in
};

// Batched tensor-core GEMM (tcgen05): modes and parameters.
enum TcMode {
    kTcGateZ = 0,       // z[t][m] fp32 (+ union bitmap) from weight rows x token rows
    kTcGateSplit = 1,   // u[t][m] as bf16 hi rows [0,npad) and lo rows [npad,2 npad)
    kTcUp = 2,          // h[t][ch] = g[t][ch] * <x[t], W_up[ch]> over the active channel blocks
    kTcDown = 3         // y[t][m] = sum over the active channel blocks of h[t][ch] * W_down[ch][m]
};

struct alignas(64) TcParams {
    CUtensorMap ta;         // A operand: weight rows, tile box 64 x 128 (down: W_down, box 64 x 64)
    CUtensorMap tb;         // B operand: token rows, tile box 64 x nb
    CUtensorMap tg;         // gather: the A weights again with a one-row box (W_up, or W_down)
    int mode;
    int m_total;            // output rows: gate rows, d_ff (up), d (down)
    int k_total;            // contraction length of gate and up
    int d_ff;               // up, down: channels (bits of the union bitmap)
    int force_all;          // up, down: every channel block (the dense FFN)
    int n, npad, nb;        // tokens, tokens padded to 16, MMA N (npad or 2 npad)
    int paired;             // accumulator columns t and npad+t are hi and lo parts
    int h_pairs;            // up: also write the lo rows of h (B of a paired down)
    float* z;               // gate: z [n][ldz]
    long long ldz;
    void* out;              // gate-split, up: bf16 [2 npad][ldo]; down: bf16 y [n][ldo]
    long long ldo;
    const float* zsel;      // up, threshold: z [n][ldsel]
    const float* gsel;      // up, top-K: gbuf [n][ldsel]
    long long ldsel;
    float tau;
    int topk;
    uint32_t* ubits;        // gate: union bitmap out (threshold), zeroed (top-K); up, down: read
    uint32_t* selbits;      // gate, threshold: per-token selection bits [n][selw] (bit k: z[t,k] > tau), or NULL
    int selw;               // words per token row of selbits (ceil(d_ff / 32))
    int gather;             // up, down: gather the union's channel rows (tg) in list order when the union is
                            // under half the channels, else read whole 128-channel blocks (ta)
    const int* ulist;       // gather: the union's channels, ascending, padded with channel 0 to a multiple of 128
    const int* ucount;      // gather: the union's size
    float* part;            // [CTAs][128][nb] each CTA's parked stream-K part (room for [CTAs][2][128][256])
    unsigned* tickets;      // two counters per tile (parts arrived, owner warps done), zero between launches
    int* status;
    int* hstatus;           // host-mapped mirror of the status word, or NULL
    int stages;             // set by the launcher
    uint32_t tmem_cols;     // set by the launcher
};


// Bits of the device status word: a bounded wait gave up, or a kernel's own
// bounds check rejected an index or a count written by an earlier kernel (the
// access was skipped).
enum StatusBits { kStatusWaitTimeout = 2, kStatusBounds = 4 };

// Set `bits` in the sticky device status word `st`, and copy the word into the
// handle's host-mapped mirror `hst` (NULL: none) with a plain system-scope
// store, so the host sees the failure on its next call without synchronising.
// Racing raisers may leave the mirror short of a bit; it is never zero after a
// raise, and the device word keeps every bit.
__device__ __forceinline__ void raise_status(int* st, int* hst, int bits) {
    const int old = st ? atomicOr(st, bits) : 0;
    if (hst) asm volatile("st.relaxed.sys.global.b32 [%0], %1;" ::"l"(hst), "r"(old | bits) : "memory");
}

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

// Launch with programmatic dependent launch (PDL) when `pdl` is set.  A
// `cooperative` launch is one whose CTAs meet at grid-wide barriers: the
// runtime then refuses a grid that cannot have all its CTAs resident at once.
template <class K, class P>
inline cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             const P& params, bool cooperative = false) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cooperative) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, params);
}

// Host-side launchers (one per kernel family); return cudaError_t.
cudaError_t launch_gate(int wdtype, const GateParams& p, int nt, int rw, int gate_kind, int grid,
                        size_t smem, cudaStream_t s, bool pdl);
size_t gate_smem_bytes(int wdtype, int nt, int d, int r, int gate_kind, int cpb, int mw);
cudaError_t launch_gate_stream(int wdtype, const GateParams& p, int nt, int gate_kind, int grid, size_t smem,
                               cudaStream_t s, bool pdl);
size_t gate_stream_smem_bytes(int nt, int d, int r, int gate_kind, int cpb, int mw, int sb, int nb);
// Largest dynamic shared memory a CTA may use on sm_100 (227 KB).
constexpr size_t kMaxSmemPerCta = 232448;
// Streaming geometry of the gate kernel for token tile nt: piece bytes *sb and
// pieces per warp *nb maximising the bytes in flight (ties: more pieces) within
// kMaxSmemPerCta; false if even two 2 KB pieces per warp do not fit.
bool gate_stream_geometry(int nt, int d, int r, int gate_kind, int cpb, int mw, int* sb, int* nb, size_t* smem);
cudaError_t launch_lopa_u(int wdtype, const LopaUParams& p, int nt, cudaStream_t s, bool pdl);
constexpr int kLopaRowsPerCta = 2;
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_down(int wdtype, const DownParams& p, int nt, int slices, size_t smem,
                        cudaStream_t s, bool pdl);
size_t down_smem_bytes(int wdtype, int nt, int nseg, int cpb);
int down_slice_cols(int wdtype);
cudaError_t launch_transpose(int wdtype, const void* src, void* dst, int rows, int cols,
                             cudaStream_t s);
bool decode_geometry(int nt, int d, int r, int gate_kind, int cpb, int mw, int vec, int grid, int* sb, int* nb,
                     size_t* smem);
cudaError_t launch_decode(int wdtype, const DecodeParams& p, int nt, int gate_kind, int grid, size_t smem,
                          cudaStream_t s, bool pdl);
constexpr int kDecodeMaxTokens = 4;   // the fused decode kernel takes up to this many tokens
constexpr int kFusedMaxTokens = 2;    // ... and is preferred to the tensor-core path up to this many
size_t tc_smem_bytes(int nb, int* stages);
cudaError_t encode_tile_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                            uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows);
cudaError_t launch_tc(const TcParams& p, int grid, cudaStream_t s, bool pdl);
// The union bitmap (bit k of word k / 32) as an ascending channel list,
// padded with channel 0 to a multiple of 128, and its size.
cudaError_t launch_union_list(const uint32_t* ubits, int d_ff, int* list, int* count, cudaStream_t s, bool pdl);
constexpr int kTcGatherMaxTokens = 8;  // batches up to this size may gather the union's rows
constexpr int kTcMaxTokens = 256;     // token columns of one tensor-core pass (MMA N <= 256)
constexpr int kTcMaxTokensLopa = 128; // ... with LoPA, whose u enters the gate as hi/lo pairs (2 x 128 columns)

}  // namespace sffn
