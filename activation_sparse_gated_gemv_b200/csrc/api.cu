// C ABI of the activation-sparse gated FFN (declared in include/sffn.h).
//
// Host-side orchestration only: argument checks, the device workspace plan,
// weight repacking, and the kernel sequence of one forward:
//   bf16, 3 tokens and more (or 2 where the decode kernel does not fit):
//               gate GEMM (z, union bitmap) [-> top-K / top-p] -> up GEMM ->
//               down GEMM on the tensor cores (LoPA: x A GEMM, then the z GEMM),
//               one pass per 128 tokens
//   threshold, 1..2 tokens (fp32: up to 4): one fused decode kernel (LoPA's
//               x A inside it)
//   otherwise:  [LoPA x A] -> gate+select+up -> down, or for top-K / top-p
//               [LoPA x A] -> gate (z) -> select -> preselected up -> down
// Every kernel is launched with programmatic dependent launch so its launch
// latency overlaps the previous kernel's tail; each kernel waits on its
// predecessor before touching shared buffers.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "common.cuh"
#include "sffn.h"

using namespace sffn;

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    const int code = e == cudaErrorMemoryAllocation ? SFFN_ERR_OOM : SFFN_ERR_CUDA;
    return fail(code, "%s: %s", what, cudaGetErrorString(e));
}

#define SFFN_CUDA(call, what)                              \
    do {                                                   \
        cudaError_t e_ = (call);                           \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

struct DeviceGuard {
    int prev = -1, dev;
    cudaError_t err = cudaSuccess;
    explicit DeviceGuard(int d) : dev(d) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) err = cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        if (prev >= 0 && prev != dev) cudaSetDevice(prev);
    }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-side fault injection for the error paths of sffn_create and
// sffn_set_weights.  The environment variable SFFN_FAULT = "alloc:N" or
// "copy:N" makes the N-th device allocation (cudaMalloc, cudaHostAlloc) or
// the N-th host-to-device copy of one such call report failure (out of
// memory, or a CUDA error) without touching the device; unset, it costs one
// getenv per call.
struct HostFaults {
    int alloc_at = 0, copy_at = 0, allocs = 0, copies = 0;
    HostFaults() {
        const char* f = std::getenv("SFFN_FAULT");
        if (!f) return;
        int n = 0;
        if (std::sscanf(f, "alloc:%d", &n) == 1) alloc_at = n;
        else if (std::sscanf(f, "copy:%d", &n) == 1) copy_at = n;
    }
    cudaError_t malloc_dev(void** p, size_t bytes) {
        if (alloc_at > 0 && ++allocs == alloc_at) return cudaErrorMemoryAllocation;
        return cudaMalloc(p, bytes);
    }
    cudaError_t malloc_host_mapped(void** p, size_t bytes) {
        if (alloc_at > 0 && ++allocs == alloc_at) return cudaErrorMemoryAllocation;
        return cudaHostAlloc(p, bytes, cudaHostAllocMapped);
    }
    cudaError_t copy(void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
        if (copy_at > 0 && ++copies == copy_at) return cudaErrorInvalidValue;
        return cudaMemcpyAsync(dst, src, bytes, kind, s);
    }
};

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Plan {
    int g1 = 0, cpb = 0, mw = 0;                          // gate grid
    int down_slices = 0, down_chunks = 0;
};

}  // namespace

struct sffn_ctx {
    sffn_config cfg{};
    int sms = 0;
    size_t esz = 0;
    void* wg = nullptr;
    void* a = nullptr;
    void* bcm = nullptr;
    void* wup = nullptr;
    void* wdn = nullptr;
    bool has_dense = false, has_lopa = false, ready = false;
    void* ws = nullptr;
    float* zbuf = nullptr;
    float* gbuf = nullptr;
    uint8_t* sel = nullptr;
    int* lst_idx = nullptr;
    float* lst_h = nullptr;
    uint32_t* lst_mask = nullptr;
    int* seg_count = nullptr;
    float* u = nullptr;
    float* dpart = nullptr;
    uint32_t* umask = nullptr;   // fused decode: [g1][ceil(cpb / 32)] union mask of each CTA's slots
    float* fpart = nullptr;      // fused decode, dense FFN: [g1][min(max_tokens, 4)][d] partials of y
    unsigned* tickets = nullptr;
    unsigned* dbar = nullptr;    // fused decode: grid-barrier arrival counters
    unsigned long long x_arrivals = 0;   // ... and the count its x counter has reached (host forwards)
    int* status = nullptr;
    int* hstat = nullptr;        // host-mapped mirror of the status word (host address)
    int* hstat_dev = nullptr;    // ... and its device address, given to the kernels
    void* xdev = nullptr;
    void* ydev = nullptr;
    // tensor-core batched path (bf16 handles with max_tokens > 1)
    bool tc = false;
    int tc_npad_max = 0;
    long long tc_ldh = 0;
    uint32_t* ubits = nullptr;
    uint32_t* selbits = nullptr; // [max_tokens][ceil(d_ff / 32)] per-token selection bits of the tensor-core gate
    int selw = 0;

    void* h2 = nullptr;          // [npad][tc_ldh] bf16: h, one row per token
    void* u2 = nullptr;          // [2 npad][r] bf16: LoPA x A as hi/lo rows (passes of up to 128 tokens)
    float* tc_part = nullptr;    // [sms][2][128][256] floats: room for one parked part per CTA at any N
    unsigned* tc_tickets = nullptr;
    bool maps_ok = false;        // weight tensor maps encoded
    CUtensorMap map_wg{}, map_at{}, map_bcm{}, map_wup{}, map_wdn{};
    bool maps_g_ok = false;      // one-row-box maps of W_up and W_down for the gathered passes
    CUtensorMap map_wup_g{}, map_wdn_g{};
    int* ulist = nullptr;        // [round_up(d_ff, 128)] the union's channels, ascending (gathered passes)
    int* ucount = nullptr;
    bool last_tc = false;        // the last forward took the tensor-core path
    bool last_topk = false;
    float last_tau = 0.f;
    Plan plan;
    int last_n = -1;
    cudaStream_t last_stream = nullptr;
    int last_launches = 0;
    const char* last_names[64] = {};
    std::vector<cudaEvent_t> events;
    uint32_t* hot = nullptr;     // heavy-hitter channel bits [ceil(d_ff / 32)] (kept once allocated)
    bool hot_on = false;         // a non-empty hot set is in force
    // one-shot injections for the failure tests (sffn_debug_inject)
    unsigned long long inj_wait_ns = 0;   // next fused decode: this wait limit, and a barrier no one completes
    bool inj_bad_index = false;           // next unfused forward: a bad list entry before the down kernel
};

namespace {

constexpr size_t kPreselSmemCap = 110 * 1024;  // keeps two up-pass CTAs per SM

int pick_nt(int n) { return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : 8; }

int presel_nt(const sffn_ctx* h, int n) {
    int nt = pick_nt(n);
    while (nt > 1 && gate_smem_bytes(h->cfg.wdtype, nt, h->cfg.d, 0, kGatePreselected, h->plan.cpb,
                                     h->plan.mw) > kPreselSmemCap)
        nt /= 2;
    return nt;
}

// Token tile and streaming geometry of the streaming gate kernel: the largest
// tile (at most the batch) for which some geometry fits; see
// gate_stream_geometry for the piece size and depth.
struct StreamGeom {
    int nt, sb, nb;
    size_t smem;
};
StreamGeom stream_geom(const sffn_ctx* h, int n, int gate_kind) {
    const sffn_config& c = h->cfg;
    const int r = gate_kind == kGateLopa ? c.lopa_rank : 0;
    StreamGeom g{pick_nt(n), 0, 0, 0};
    while (!gate_stream_geometry(g.nt, c.d, r, gate_kind, h->plan.cpb, h->plan.mw, &g.sb, &g.nb, &g.smem) &&
           g.nt > 1)
        g.nt /= 2;
    return g;
}

// Stage events are recorded as external event nodes under stream capture so
// that a replayed graph still timestamps them.
// Name of launch i of the forward (for profiles and timing reports).
void set_name(sffn_ctx* h, int i, const char* name) {
    if (i < 64) h->last_names[i] = name;
}

void record(sffn_ctx* h, int i, cudaStream_t s) {
    if (i >= (int)h->events.size()) return;
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(h->events[i], s, cudaEventRecordExternal);
    else
        cudaEventRecord(h->events[i], s);
}

// The status word's bits as a return code: a failed bounds check before a
// timed-out wait.
int status_code(int st) {
    if (st & kStatusBounds) return fail(SFFN_ERR_DEVICE_CHECK, "a kernel's bounds check failed (status 0x%x)", st);
    if (st & kStatusWaitTimeout) return fail(SFFN_ERR_TIMEOUT, "a bounded device wait timed out (status 0x%x)", st);
    if (st) return fail(SFFN_ERR_DEVICE_CHECK, "device status word 0x%x", st);
    return SFFN_OK;
}

// The host-mapped mirror of the status word, read without synchronising: set
// once a kernel of an earlier forward that has finished raised a bit.
int mirrored_status(const sffn_ctx* h) {
    return h->hstat ? *reinterpret_cast<volatile const int*>(h->hstat) : 0;
}

int check_select(const sffn_ctx* h, const sffn_select* sel) {
    if (!sel) return fail(SFFN_ERR_INVALID_ARG, "sel is NULL");
    if (sel->kind == SFFN_SELECT_THRESHOLD) {
        if (std::isnan(sel->tau) || (std::isinf(sel->tau) && sel->tau < 0))
            return fail(SFFN_ERR_INVALID_ARG, "threshold tau must be a number or +inf");
    } else if (sel->kind == SFFN_SELECT_TOPK) {
        if (sel->k < 0 || sel->k > h->cfg.d_ff)
            return fail(SFFN_ERR_INVALID_ARG, "top-K k=%d outside [0, d_ff=%d]", sel->k, h->cfg.d_ff);
    } else if (sel->kind == SFFN_SELECT_TOPP) {
        if (!(sel->p >= 0.f && sel->p <= 1.f))
            return fail(SFFN_ERR_INVALID_ARG, "top-p p=%g outside [0, 1]", (double)sel->p);
    } else {
        return fail(SFFN_ERR_INVALID_ARG, "unknown select kind %d", sel->kind);
    }
    return SFFN_OK;
}

int check_forward(const sffn_ctx* h, const void* x, int n, int gate_mode, const sffn_select* sel,
                  const void* out, bool device_ptrs) {
    if (!h) return fail(SFFN_ERR_INVALID_ARG, "handle is NULL");
    if (const int st = mirrored_status(h)) return status_code(st);
    if (n < 0 || n > h->cfg.max_tokens)
        return fail(SFFN_ERR_INVALID_ARG, "n_tokens=%d outside [0, max_tokens=%d]", n, h->cfg.max_tokens);
    if (gate_mode != SFFN_GATE_DENSE && gate_mode != SFFN_GATE_LOPA)
        return fail(SFFN_ERR_INVALID_ARG, "unknown gate mode %d", gate_mode);
    const int rc = check_select(h, sel);
    if (rc) return rc;
    if (n > 0) {
        if (!x || !out) return fail(SFFN_ERR_INVALID_ARG, "x or out is NULL");
        if (device_ptrs && (!aligned16(x) || !aligned16(out)))
            return fail(SFFN_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
    }
    if (!h->ready) return fail(SFFN_ERR_NOT_READY, "sffn_set_weights has not been called");
    if (gate_mode == SFFN_GATE_DENSE && !h->has_dense)
        return fail(SFFN_ERR_UNSUPPORTED, "dense gate requested but no W_gate was set");
    if (gate_mode == SFFN_GATE_LOPA && !h->has_lopa)
        return fail(SFFN_ERR_UNSUPPORTED, "LoPA gate requested but A and B were not set");
    return SFFN_OK;
}

// Batched forward on the tensor cores: gate GEMM -> [top-K] -> up GEMM ->
// down GEMM, every GEMM one stream-K tcgen05 kernel over all SMs; the up and
// down kernels find the active channel blocks in the gate's union bitmap.
// Returns SFFN_ERR_UNSUPPORTED (nothing launched) when a tensor map cannot be
// made for this call; the caller then takes the CUDA-core path.
int run_tc(sffn_ctx* h, const void* x, int n, bool lopa, const sffn_select* sel, void* out, cudaStream_t s,
           bool dense, int& launches, int t0) {
    const sffn_config& c = h->cfg;
    const bool topk = sel->kind != SFFN_SELECT_THRESHOLD;   // a top-K or top-p mask decides
    const int npad = (int)round_up(n, 16);
    const float tau = topk ? 0.f : sel->tau;
    if (!h->maps_ok || (lopa && c.lopa_rank < 64)) return SFFN_ERR_UNSUPPORTED;
    CUtensorMap map_x{}, map_u2{}, map_h2{};
    if (encode_tile_map(&map_x, x, c.d, n, (uint64_t)c.d * 2, 64, npad) != cudaSuccess ||
        encode_tile_map(&map_h2, h->h2, h->tc_ldh, npad, (uint64_t)h->tc_ldh * 2, 64, npad) != cudaSuccess ||
        (lopa && encode_tile_map(&map_u2, h->u2, c.lopa_rank, 2 * npad, (uint64_t)c.lopa_rank * 2, 64, 2 * npad) !=
                     cudaSuccess))
        return SFFN_ERR_UNSUPPORTED;

    TcParams base{};
    base.n = n;
    base.npad = npad;
    base.tau = tau;
    base.topk = topk ? 1 : 0;
    base.part = h->tc_part;
    base.tickets = h->tc_tickets;
    base.status = h->status;
    base.hstatus = h->hstat_dev;

    TcParams g = base;
    g.mode = kTcGateZ;
    float* zrows = h->zbuf + (size_t)t0 * c.d_ff;      // this pass's tokens' rows of the workspace
    float* grows = h->gbuf + (size_t)t0 * c.d_ff;
    uint8_t* srows = h->sel + (size_t)t0 * c.d_ff;
    g.z = zrows;
    g.ldz = c.d_ff;
    g.ubits = h->ubits;
    g.selbits = topk ? nullptr : h->selbits + (size_t)t0 * h->selw;
    g.selw = h->selw;
    g.m_total = c.d_ff;
    if (lopa) {
        TcParams u = base;                      // u = x A, as hi/lo bf16 rows
        u.mode = kTcGateSplit;
        u.ta = h->map_at; u.tb = map_x;
        u.m_total = c.lopa_rank; u.k_total = c.d; u.nb = npad;
        u.out = h->u2; u.ldo = c.lopa_rank;
        SFFN_CUDA(launch_tc(u, h->sms, s, true), "tensor-core x A launch");
        set_name(h, launches, "tc_lopa_u");
        record(h, ++launches, s);
        g.ta = h->map_bcm; g.tb = map_u2;
        g.k_total = c.lopa_rank; g.nb = 2 * npad; g.paired = 1;
    } else {
        g.ta = h->map_wg; g.tb = map_x;
        g.k_total = c.d; g.nb = npad;
    }
    SFFN_CUDA(launch_tc(g, h->sms, s, true), "tensor-core gate launch");
    set_name(h, launches, "tc_gate");
    record(h, ++launches, s);

    if (topk) {
        TopkParams tp{};
        tp.zbuf = zrows; tp.n = n; tp.d_ff = c.d_ff; tp.k = sel->k; tp.gbuf = grows; tp.sel = srows;
        tp.ubits = h->ubits;
        tp.mode = sel->kind == SFFN_SELECT_TOPP ? 1 : 0;
        tp.p = sel->p;
        SFFN_CUDA(launch_topk(tp, s, true), "top-K / top-p launch");
        set_name(h, launches, tp.mode ? "topp" : "topk");
        record(h, ++launches, s);
    }

    // Small batches: the up and down passes gather exactly the union's rows
    // (a list built from the union bitmap); larger ones, whose union covers
    // nearly every channel, read whole 128-channel blocks.
    const bool gather = !dense && n <= kTcGatherMaxTokens && h->maps_g_ok;
    if (gather) {
        SFFN_CUDA(launch_union_list(h->ubits, c.d_ff, h->ulist, h->ucount, s, true), "union list launch");
        set_name(h, launches, "union_list");
        record(h, ++launches, s);
    }

    TcParams w = base;                          // h = g * <x, W_up[ch]> over the active channel blocks
    w.mode = kTcUp;
    w.ta = h->map_wup; w.tg = h->map_wup_g; w.tb = map_x;
    w.gather = gather ? 1 : 0; w.ulist = h->ulist; w.ucount = h->ucount;
    w.ubits = h->ubits; w.d_ff = c.d_ff; w.force_all = dense ? 1 : 0;
    w.m_total = c.d_ff; w.k_total = c.d; w.nb = npad;
    // h goes to the down pass as one bf16 row per token: its rounding moves y by
    // about 2^-9 relative (LoPA's u, which decides selections, keeps hi/lo pairs)
    w.out = h->h2; w.ldo = h->tc_ldh; w.h_pairs = 0;
    w.zsel = zrows; w.gsel = grows; w.ldsel = c.d_ff;
    SFFN_CUDA(launch_tc(w, h->sms, s, true), "tensor-core up launch");
    set_name(h, launches, "tc_up");
    record(h, ++launches, s);

    TcParams dn = base;                         // y = sum over the active blocks of h W_down[ch]
    dn.mode = kTcDown;
    dn.ta = h->map_wdn; dn.tg = h->map_wdn_g; dn.tb = map_h2;
    dn.gather = gather ? 1 : 0; dn.ulist = h->ulist; dn.ucount = h->ucount;
    dn.ubits = h->ubits; dn.d_ff = c.d_ff; dn.force_all = dense ? 1 : 0;
    dn.m_total = c.d; dn.nb = npad; dn.paired = 0;
    dn.out = out; dn.ldo = c.d;
    SFFN_CUDA(launch_tc(dn, h->sms, s, true), "tensor-core down launch");
    set_name(h, launches, "tc_down");
    record(h, ++launches, s);

    h->last_n = n;
    h->last_stream = s;
    h->last_launches = launches;
    h->last_tc = true;
    h->last_topk = topk;
    h->last_tau = tau;
    return SFFN_OK;
}

// xmapped: a forward with host buffers whose x is page-locked host memory the
// device can address (x is then the device buffer it goes to): the fused
// decode kernel pulls it in itself; the other paths copy it first.
int run_forward(sffn_ctx* h, const void* x, int n, int gate_mode, const sffn_select* sel, void* out,
                cudaStream_t s, bool dense, const void* xmapped = nullptr) {
    const sffn_config& c = h->cfg;
    const Plan& P = h->plan;
    const bool lopa = gate_mode == SFFN_GATE_LOPA;
    const int gk = lopa ? kGateLopa : kGateDense;
    const bool pdl = true;
    int launches = 0;
    record(h, 0, s);
    for (auto& nm : h->last_names) nm = nullptr;

    // Fused decode path: threshold selection, a few tokens; the sparse forward,
    // or the dense FFN with a dense gate.
    int dec_sb = 0, dec_nb = 0;
    size_t dec_smem = 0;
    const int dec_nt = pick_nt(n);
    const bool fused = sel->kind == SFFN_SELECT_THRESHOLD && !(dense && lopa) && n <= kDecodeMaxTokens &&
                       decode_geometry(dec_nt, c.d, lopa ? c.lopa_rank : 0, gk, P.cpb, P.mw,
                                       c.wdtype == SFFN_BF16 ? 8 : 4, P.g1, &dec_sb, &dec_nb,
                                       &dec_smem);

    h->last_tc = false;
    if (xmapped && !fused)
        SFFN_CUDA(cudaMemcpyAsync(const_cast<void*>(x), xmapped, (size_t)n * c.d * h->esz, cudaMemcpyDefault, s),
                  "x host-to-device copy");
    // Three or more tokens: the tensor-core path (measured faster than the fused
    // decode kernel from n = 3 on every shape but one); one or two: the fused
    // decode kernel, or the tensor-core path for two tokens where the decode
    // kernel's shared memory does not fit.
    if (h->tc && (n > kFusedMaxTokens || (n > 1 && !fused))) {
        // More tokens than one pass takes (256, or 128 with LoPA): one
        // tensor-core pass per block of tokens (each pass streams the weights
        // again, which still beats the CUDA-core path's fp32 arithmetic).
        const int pass = lopa ? kTcMaxTokensLopa : kTcMaxTokens;
        int rc = SFFN_OK;
        for (int t0 = 0; t0 < n && rc == SFFN_OK; t0 += pass) {
            const int nc = n - t0 < pass ? n - t0 : pass;
            rc = run_tc(h, static_cast<const char*>(x) + (size_t)t0 * c.d * h->esz, nc, lopa, sel,
                        static_cast<char*>(out) + (size_t)t0 * c.d * h->esz, s, dense, launches, t0);
            if (rc == SFFN_ERR_UNSUPPORTED && t0 > 0) rc = fail(SFFN_ERR_CUDA, "tensor-core pass failed mid-batch");
        }
        if (rc != SFFN_ERR_UNSUPPORTED) {
            h->last_n = n;
            return rc;
        }
    }

    if (lopa && !fused) {
        LopaUParams lp{};
        lp.x = x; lp.at = h->a; lp.n = n; lp.d = c.d; lp.r = c.lopa_rank; lp.u = h->u;
        SFFN_CUDA(launch_lopa_u(c.wdtype, lp, pick_nt(n), s, pdl), "LoPA x*A launch");
        set_name(h, launches, "lopa_u");
        record(h, ++launches, s);
    }

    if (fused) {
        DecodeParams dp{};
        dp.x = x; dp.n = n; dp.d = c.d; dp.d_ff = c.d_ff; dp.r = c.lopa_rank;
        dp.wg = h->wg; dp.bcm = h->bcm; dp.at = h->a; dp.u = h->u; dp.wup = h->wup; dp.wdn = h->wdn;
        dp.tau = sel->tau; dp.cpb = P.cpb; dp.mw = P.mw;
        dp.lst_idx = h->lst_idx; dp.lst_h = h->lst_h; dp.lst_mask = h->lst_mask; dp.seg_count = h->seg_count;
        dp.sb = dec_sb; dp.nb = dec_nb; dp.status = h->status; dp.hstatus = h->hstat_dev; dp.umask = h->umask; dp.part = h->fpart;
        dp.wait_ns = h->inj_wait_ns ? h->inj_wait_ns : kWaitLimitNs;
        dp.bar_extra = h->inj_wait_ns ? 1 : 0;
        h->inj_wait_ns = 0;
        dp.tickets = h->dbar; dp.y = out; dp.hot = h->hot_on && !dense ? h->hot : nullptr;
        dp.dense = dense ? 1 : 0;
        // The sparse forward's down projection: each CTA's own rows into a
        // partial of y (measured faster up to d = 4096), or the union gather by
        // column slice (faster on the 70B shape, d = 8192).
        dp.own_rows = c.d <= 4096 ? 1 : 0;
        if (xmapped) {
            dp.xh = xmapped;
            dp.xld = (int)(((size_t)n * c.d * h->esz + 8191) / 8192);
            dp.xtarget = h->x_arrivals + (unsigned long long)dp.xld;
        }
        SFFN_CUDA(launch_decode(c.wdtype, dp, dec_nt, gk, P.g1, dec_smem, s, pdl), "fused decode launch");
        if (xmapped) h->x_arrivals = dp.xtarget;          // counted only once the launch is in
        set_name(h, launches, dense ? "decode_dense" : "decode_fused");
        record(h, ++launches, s);
        h->last_n = n;
        h->last_stream = s;
        h->last_launches = launches;
        return SFFN_OK;
    }

    GateParams gp{};
    gp.x = x; gp.n = n; gp.d = c.d; gp.d_ff = c.d_ff; gp.r = c.lopa_rank;
    gp.wg = h->wg; gp.bcm = h->bcm; gp.u = h->u; gp.wup = h->wup; gp.wdn = h->wdn;
    gp.force_all = dense ? 1 : 0;
    gp.tau = sel->tau;
    gp.zbuf = h->zbuf; gp.gbuf = h->gbuf; gp.sel = h->sel;
    gp.cpb = P.cpb; gp.mw = P.mw;
    gp.lst_idx = h->lst_idx; gp.lst_h = h->lst_h; gp.lst_mask = h->lst_mask; gp.seg_count = h->seg_count;

    const StreamGeom sg = stream_geom(h, n, gk);
    if (sg.sb == 0) return fail(SFFN_ERR_UNSUPPORTED, "d=%d too large for the streaming gate's shared memory", c.d);
    gp.sb = sg.sb;
    gp.nb = sg.nb;
    gp.status = h->status;
    gp.hstatus = h->hstat_dev;
    if (sel->kind == SFFN_SELECT_THRESHOLD) {
        gp.out = kOutSelectUp;
        SFFN_CUDA(launch_gate_stream(c.wdtype, gp, sg.nt, gk, P.g1, sg.smem, s, pdl), "gate/select/up launch");
        set_name(h, launches, "gate_select_up");
        record(h, ++launches, s);
    } else {
        gp.out = kOutWriteZ;
        SFFN_CUDA(launch_gate_stream(c.wdtype, gp, sg.nt, gk, P.g1, sg.smem, s, pdl), "gate launch");
        set_name(h, launches, "gate_z");
        record(h, ++launches, s);
        TopkParams tp{};
        tp.zbuf = h->zbuf; tp.n = n; tp.d_ff = c.d_ff; tp.k = sel->k; tp.gbuf = h->gbuf; tp.sel = h->sel;
        tp.mode = sel->kind == SFFN_SELECT_TOPP ? 1 : 0;
        tp.p = sel->p;
        SFFN_CUDA(launch_topk(tp, s, pdl), "top-K / top-p launch");
        set_name(h, launches, tp.mode ? "topp" : "topk");
        record(h, ++launches, s);
        gp.out = kOutSelectUp;
        const int nt = presel_nt(h, n);
        SFFN_CUDA(launch_gate(c.wdtype, gp, nt, 1, kGatePreselected, P.g1,
                              gate_smem_bytes(c.wdtype, nt, c.d, 0, kGatePreselected, P.cpb, P.mw), s, pdl),
                  "selected up launch");
        set_name(h, launches, "preselected_up");
        record(h, ++launches, s);
    }

    DownParams dp{};
    dp.wdn = h->wdn; dp.n = n; dp.d = c.d; dp.d_ff = c.d_ff;
    dp.seg_count = h->seg_count; dp.g1 = P.g1; dp.cpb = P.cpb;
    dp.lst_idx = h->lst_idx; dp.lst_h = h->lst_h; dp.part = h->dpart;
    dp.tickets = h->tickets; dp.y = out;
    dp.chunks = P.down_chunks;
    dp.status = h->status;
    dp.hstatus = h->hstat_dev;
    if (h->inj_bad_index) {
        // failure test: a list entry outside its segment and a count beyond its
        // segment's slots, written by the host between the gate and the down
        // kernel; the down kernel's checks must catch both
        h->inj_bad_index = false;
        const int bad_idx = c.d_ff + 7, bad_cnt = P.cpb + 5;
        SFFN_CUDA(cudaMemcpyAsync(h->lst_idx, &bad_idx, sizeof bad_idx, cudaMemcpyHostToDevice, s), "inject");
        if (P.g1 > 1)
            SFFN_CUDA(cudaMemcpyAsync(h->seg_count + 1, &bad_cnt, sizeof bad_cnt, cudaMemcpyHostToDevice, s),
                      "inject");
    }
    const int dnt = pick_nt(n);
    const int nseg = (P.g1 + P.down_chunks - 1) / P.down_chunks;
    SFFN_CUDA(launch_down(c.wdtype, dp, dnt, P.down_slices, down_smem_bytes(c.wdtype, dnt, nseg, P.cpb), s, pdl),
              "down launch");
    set_name(h, launches, "down");
    record(h, ++launches, s);

    h->last_n = n;
    h->last_stream = s;
    h->last_launches = launches;
    return SFFN_OK;
}

int forward_common(sffn_handle h, const void* x, int n, int gate_mode, const sffn_select* sel, void* out,
                   void* stream, bool dense) {
    int rc = check_forward(h, x, n, gate_mode, sel, out, true);
    if (rc) return rc;
    if (n == 0) return SFFN_OK;
    DeviceGuard g(h->cfg.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    return run_forward(h, x, n, gate_mode, sel, out, static_cast<cudaStream_t>(stream), dense);
}

void free_weights(sffn_ctx* h) {
    for (void** p : {&h->wg, &h->a, &h->bcm, &h->wup, &h->wdn}) {
        if (*p) cudaFree(*p);
        *p = nullptr;
    }
    h->has_dense = h->has_lopa = h->ready = false;
}

}  // namespace

extern "C" {

const char* sffn_strerror(int code) {
    switch (code) {
        case SFFN_OK: return "ok";
        case SFFN_ERR_INVALID_ARG: return "invalid argument";
        case SFFN_ERR_NOT_READY: return "weights not set";
        case SFFN_ERR_UNSUPPORTED: return "unsupported mode for this handle";
        case SFFN_ERR_CUDA: return "CUDA error";
        case SFFN_ERR_OOM: return "out of device memory";
        case SFFN_ERR_TIMEOUT: return "device wait timed out";
        case SFFN_ERR_DEVICE_CHECK: return "a kernel's own bounds check failed";
        default: return "unknown status";
    }
}

const char* sffn_last_error(void) { return g_err; }

int sffn_create(sffn_handle* out, const sffn_config* cfg) {
    if (!out || !cfg) return fail(SFFN_ERR_INVALID_ARG, "out or cfg is NULL");
    *out = nullptr;
    const sffn_config c = *cfg;
    if (c.d <= 0 || c.d % 8 || c.d_ff <= 0 || c.lopa_rank < 0 || c.lopa_rank % 8 ||
        c.max_tokens < 1 || c.max_tokens > kMaxTokens || (c.wdtype != SFFN_BF16 && c.wdtype != SFFN_F32))
        return fail(SFFN_ERR_INVALID_ARG,
                    "bad config d=%d d_ff=%d r=%d max_tokens=%d wdtype=%d (d, r multiples of 8; "
                    "1 <= max_tokens <= %d)", c.d, c.d_ff, c.lopa_rank, c.max_tokens, c.wdtype, kMaxTokens);
    if ((long long)c.d * c.d_ff > (1LL << 31) - 1 || c.lopa_rank > 4096)
        return fail(SFFN_ERR_INVALID_ARG, "shape too large");
    int ndev = 0;
    SFFN_CUDA(cudaGetDeviceCount(&ndev), "cudaGetDeviceCount");
    if (c.device < 0 || c.device >= ndev) return fail(SFFN_ERR_INVALID_ARG, "no CUDA device %d", c.device);
    DeviceGuard g(c.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    HostFaults faults;

    sffn_ctx* h = new (std::nothrow) sffn_ctx();
    if (!h) return fail(SFFN_ERR_OOM, "host allocation failed");
    h->cfg = c;
    h->esz = c.wdtype == SFFN_BF16 ? 2 : 4;
    cudaError_t e = cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, c.device);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "device attribute"); }

    Plan& P = h->plan;
    P.cpb = (c.d_ff + h->sms - 1) / h->sms;           // one gate CTA per SM
    P.g1 = (c.d_ff + P.cpb - 1) / P.cpb;
    P.mw = (c.max_tokens + 31) / 32;
    P.down_slices = (c.d + down_slice_cols(c.wdtype) - 1) / down_slice_cols(c.wdtype);
    P.down_chunks = h->sms / P.down_slices;                 // about one down CTA per SM
    // ... but at least 128 channels per chunk: the last CTA of a slice adds the
    // chunks' partials one after another (a 1024-channel FFN cut into 147
    // chunks of 7 took 138 us there for 8 tokens)
    if (P.down_chunks > (c.d_ff + 127) / 128) P.down_chunks = (c.d_ff + 127) / 128;
    if (P.down_chunks < 1) P.down_chunks = 1;
    if (P.down_chunks > P.g1) P.down_chunks = P.g1;

    const size_t T = c.max_tokens, F = c.d_ff, D = c.d, R = c.lopa_rank;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = round_up(off + bytes, 256); return o; };
    const size_t o_z = take(T * F * 4), o_g = take(T * F * 4), o_sel = take(T * F);
    const size_t o_idx = take(F * 4), o_h = take(F * T * 4), o_mask = take(F * P.mw * 4);
    const size_t o_seg = take((size_t)P.g1 * 4);
    const size_t o_u = take(T * R * 4);
    const size_t o_dp = take((size_t)P.down_chunks * T * D * 4);
    const size_t o_um = take((size_t)P.g1 * ((P.cpb + 31) / 32) * 4);
    const size_t o_fp = take((size_t)P.g1 * (T < kDecodeMaxTokens ? T : kDecodeMaxTokens) * D * 4);
    const size_t o_tk = take((size_t)(P.down_slices > 2 ? P.down_slices : 2) * 4), o_st = take(4);
    const size_t o_db = take(32);   // the decode kernel's grid-barrier counters (64-bit, never reset)
    const size_t o_x = take(T * D * h->esz), o_y = take(T * D * h->esz);
    // tensor-core path buffers
    h->tc = c.wdtype == SFFN_BF16 && c.max_tokens > 1;
    h->tc_npad_max = (int)round_up(c.max_tokens < kTcMaxTokens ? c.max_tokens : kTcMaxTokens, 16);
    h->tc_ldh = (long long)round_up(F, 128);
    const size_t NP = h->tc ? (size_t)h->tc_npad_max : 0;
    const size_t FDR = F > D ? (F > R ? F : R) : (D > R ? D : R);
    const size_t tiles = round_up(FDR, 128) / 128 + 1;
    const size_t o_ub = take(h->tc ? tiles * 4 * 4 : 0);
    h->selw = (int)((F + 31) / 32);
    const size_t o_sb = take(h->tc ? T * (size_t)h->selw * 4 : 0);
    const size_t NPL = NP < (size_t)kTcMaxTokensLopa ? NP : (size_t)kTcMaxTokensLopa;
    const size_t o_h2 = take(NP * (size_t)h->tc_ldh * 2), o_u2 = take(2 * NPL * R * 2);
    const size_t o_ul = take(h->tc ? (size_t)h->tc_ldh * 4 : 0), o_uc = take(h->tc ? 16 : 0);
    // stream-K partial tiles: two slots per CTA of up to 256 accumulator columns x 128 rows
    const size_t o_tp = take(h->tc ? (size_t)h->sms * 2 * 256 * 128 * 4 : 0), o_tt = take(h->tc ? tiles * 8 : 0);
    e = faults.malloc_dev(&h->ws, off);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "workspace allocation"); }
    void* hs = nullptr;
    e = faults.malloc_host_mapped(&hs, 64);
    if (e == cudaSuccess) {
        h->hstat = static_cast<int*>(hs);
        *h->hstat = 0;
        void* hd = nullptr;
        e = cudaHostGetDevicePointer(&hd, hs, 0);
        h->hstat_dev = static_cast<int*>(hd);
    }
    if (e != cudaSuccess) {
        if (h->hstat) cudaFreeHost(h->hstat);
        cudaFree(h->ws);
        delete h;
        return cuda_fail(e, "status mirror allocation");
    }
    char* b = static_cast<char*>(h->ws);
    h->zbuf = reinterpret_cast<float*>(b + o_z);
    h->gbuf = reinterpret_cast<float*>(b + o_g);
    h->sel = reinterpret_cast<uint8_t*>(b + o_sel);
    h->lst_idx = reinterpret_cast<int*>(b + o_idx);
    h->lst_h = reinterpret_cast<float*>(b + o_h);
    h->lst_mask = reinterpret_cast<uint32_t*>(b + o_mask);
    h->seg_count = reinterpret_cast<int*>(b + o_seg);
    h->u = reinterpret_cast<float*>(b + o_u);
    h->dpart = reinterpret_cast<float*>(b + o_dp);
    h->umask = reinterpret_cast<uint32_t*>(b + o_um);
    h->fpart = reinterpret_cast<float*>(b + o_fp);
    h->tickets = reinterpret_cast<unsigned*>(b + o_tk);
    h->dbar = reinterpret_cast<unsigned*>(b + o_db);
    h->status = reinterpret_cast<int*>(b + o_st);
    h->xdev = b + o_x;
    h->ydev = b + o_y;
    if (h->tc) {
        h->ubits = reinterpret_cast<uint32_t*>(b + o_ub);
        h->selbits = reinterpret_cast<uint32_t*>(b + o_sb);
        h->ulist = reinterpret_cast<int*>(b + o_ul);
        h->ucount = reinterpret_cast<int*>(b + o_uc);
        h->h2 = b + o_h2;
        h->u2 = b + o_u2;
        h->tc_part = reinterpret_cast<float*>(b + o_tp);
        h->tc_tickets = reinterpret_cast<unsigned*>(b + o_tt);
    }
    e = cudaMemset(h->ws, 0, off);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFreeHost(h->hstat);
        cudaFree(h->ws);
        delete h;
        return cuda_fail(e, "workspace init");
    }
    *out = h;
    return SFFN_OK;
}

int sffn_set_weights(sffn_handle h, const void* w_gate, const void* A, const void* B, const void* w_up,
                     const void* w_down, int src_is_device, void* stream) {
    if (!h) return fail(SFFN_ERR_INVALID_ARG, "handle is NULL");
    const sffn_config& c = h->cfg;
    if (!w_up || !w_down) return fail(SFFN_ERR_INVALID_ARG, "w_up and w_down are required");
    if (!w_gate && !(A && B)) return fail(SFFN_ERR_INVALID_ARG, "need w_gate or both A and B");
    if ((A != nullptr) != (B != nullptr)) return fail(SFFN_ERR_INVALID_ARG, "A and B go together");
    if (A && c.lopa_rank <= 0) return fail(SFFN_ERR_INVALID_ARG, "A and B need lopa_rank > 0");
    if (src_is_device)
        for (const void* p : {w_gate, A, B, w_up, w_down})
            if (p && !aligned16(p)) return fail(SFFN_ERR_INVALID_ARG, "device weights must be 16-byte aligned");
    DeviceGuard g(c.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SFFN_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    free_weights(h);
    HostFaults faults;

    const size_t big = (size_t)c.d * c.d_ff * h->esz;
    const size_t r_d = (size_t)c.lopa_rank * c.d * h->esz, r_ff = (size_t)c.lopa_rank * c.d_ff * h->esz;
    void* staging = nullptr;
    int rc = SFFN_OK;
    auto stage = [&](const void* src, size_t bytes) -> const void* {
        if (src_is_device) return src;
        if (faults.copy(staging, src, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return nullptr;
        return staging;
    };
    auto alloc = [&](void** p, size_t bytes) { return faults.malloc_dev(p, bytes); };
    cudaError_t e = cudaSuccess;
    // a failed staging copy: the runtime's error, or the injected one
    auto copy_error = [&]() {
        const cudaError_t le = cudaGetLastError();
        return le != cudaSuccess ? le : cudaErrorInvalidValue;
    };
    do {
        if (!src_is_device && (e = alloc(&staging, big > r_ff ? big : r_ff)) != cudaSuccess) break;
        if ((e = alloc(&h->wup, big)) != cudaSuccess) break;
        if ((e = alloc(&h->wdn, big)) != cudaSuccess) break;
        const void* src = stage(w_up, big);
        if (!src) { e = copy_error(); break; }
        if ((e = launch_transpose(c.wdtype, src, h->wup, c.d, c.d_ff, s)) != cudaSuccess) break;
        if ((e = cudaStreamSynchronize(s)) != cudaSuccess) break;
        if ((e = faults.copy(h->wdn, w_down, big, src_is_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                             s)) != cudaSuccess)
            break;
        if (w_gate) {
            if ((e = alloc(&h->wg, big)) != cudaSuccess) break;
            src = stage(w_gate, big);
            if (!src) { e = copy_error(); break; }
            if ((e = launch_transpose(c.wdtype, src, h->wg, c.d, c.d_ff, s)) != cudaSuccess) break;
            if ((e = cudaStreamSynchronize(s)) != cudaSuccess) break;
        }
        if (A) {
            if ((e = alloc(&h->a, r_d)) != cudaSuccess) break;
            if ((e = alloc(&h->bcm, r_ff)) != cudaSuccess) break;
            src = stage(A, r_d);
            if (!src) { e = copy_error(); break; }
            if ((e = launch_transpose(c.wdtype, src, h->a, c.d, c.lopa_rank, s)) != cudaSuccess) break;
            if ((e = cudaStreamSynchronize(s)) != cudaSuccess) break;
            src = stage(B, r_ff);
            if (!src) { e = copy_error(); break; }
            if ((e = launch_transpose(c.wdtype, src, h->bcm, c.lopa_rank, c.d_ff, s)) != cudaSuccess) break;
        }
        e = cudaStreamSynchronize(s);
    } while (0);
    if (staging) cudaFree(staging);
    if (e != cudaSuccess) {
        rc = cuda_fail(e, "sffn_set_weights");
        free_weights(h);
        return rc;
    }
    h->has_dense = w_gate != nullptr;
    h->has_lopa = A != nullptr;
    h->ready = true;
    // tensor maps of the weights for the batched tensor-core path (host-side encoding only)
    h->maps_ok = h->maps_g_ok = false;
    if (h->tc && c.d >= 64) {
        const uint64_t F = c.d_ff, D = c.d, R = c.lopa_rank;
        bool ok = encode_tile_map(&h->map_wup, h->wup, D, F, D * 2, 64, 128) == cudaSuccess &&
                  encode_tile_map(&h->map_wdn, h->wdn, D, F, D * 2, 64, 64) == cudaSuccess;
        if (ok && h->wg) ok = encode_tile_map(&h->map_wg, h->wg, D, F, D * 2, 64, 128) == cudaSuccess;
        if (ok && h->a && R >= 64)
            ok = encode_tile_map(&h->map_at, h->a, D, R, D * 2, 64, 128) == cudaSuccess &&
                 encode_tile_map(&h->map_bcm, h->bcm, R, F, R * 2, 64, 128) == cudaSuccess;
        h->maps_ok = ok;
        h->maps_g_ok = ok && encode_tile_map(&h->map_wup_g, h->wup, D, F, D * 2, 64, 1) == cudaSuccess &&
                       encode_tile_map(&h->map_wdn_g, h->wdn, D, F, D * 2, 64, 1) == cudaSuccess;
    }
    return SFFN_OK;
}

int sffn_forward(sffn_handle h, const void* x, int n_tokens, int gate_mode, const sffn_select* sel, void* out,
                 void* stream) {
    return forward_common(h, x, n_tokens, gate_mode, sel, out, stream, false);
}

int sffn_forward_dense(sffn_handle h, const void* x, int n_tokens, int gate_mode, const sffn_select* sel,
                       void* out, void* stream) {
    return forward_common(h, x, n_tokens, gate_mode, sel, out, stream, true);
}

int sffn_forward_host(sffn_handle h, const void* x_host, int n_tokens, int gate_mode, const sffn_select* sel,
                      void* out_host, void* stream) {
    int rc = check_forward(h, x_host, n_tokens, gate_mode, sel, out_host, false);
    if (rc) return rc;
    if (n_tokens == 0) return SFFN_OK;
    DeviceGuard g(h->cfg.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)n_tokens * h->cfg.d * h->esz;
    // A page-locked output that the device can address (any cudaHostAlloc'd or
    // registered buffer under unified addressing) is written by the fused
    // decode kernel itself, one slice store per CTA: no device-to-host copy.
    // Other outputs, and batches that take the multi-kernel paths, go through
    // the workspace and a copy.
    // (The check runs on every call: a buffer can be freed and its address reused.)
    void* ydst = h->ydev;
    if (n_tokens <= kFusedMaxTokens) {
        cudaPointerAttributes pa{};
        if (cudaPointerGetAttributes(&pa, out_host) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
            pa.devicePointer && aligned16(pa.devicePointer))
            ydst = pa.devicePointer;
        cudaGetLastError();
    }
    // x: page-locked host memory the device can address is pulled in by the
    // fused decode kernel itself (no copy-engine round trip); other memory is
    // copied first.
    const void* xmapped = nullptr;
    if (n_tokens <= kFusedMaxTokens && (bytes & 15) == 0) {
        cudaPointerAttributes pa{};
        if (cudaPointerGetAttributes(&pa, x_host) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
            pa.devicePointer && aligned16(pa.devicePointer))
            xmapped = pa.devicePointer;
        cudaGetLastError();
    }
    if (!xmapped)
        SFFN_CUDA(cudaMemcpyAsync(h->xdev, x_host, bytes, cudaMemcpyHostToDevice, s), "x host-to-device copy");
    rc = run_forward(h, h->xdev, n_tokens, gate_mode, sel, ydst, s, false, xmapped);
    if (rc) return rc;
    if (ydst == h->ydev)
        SFFN_CUDA(cudaMemcpyAsync(out_host, h->ydev, bytes, cudaMemcpyDeviceToHost, s), "y device-to-host copy");
    SFFN_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    return SFFN_OK;
}

int sffn_check_status(sffn_handle h) {
    if (!h) return fail(SFFN_ERR_INVALID_ARG, "handle is NULL");
    DeviceGuard g(h->cfg.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    SFFN_CUDA(cudaDeviceSynchronize(), "device synchronize");
    int st = 0;
    SFFN_CUDA(cudaMemcpy(&st, h->status, sizeof st, cudaMemcpyDeviceToHost), "status read");
    return status_code(st);
}

int sffn_get_active(sffn_handle h, int32_t* idx, int32_t* counts, int32_t* union_size) {
    if (!h || !idx || !counts) return fail(SFFN_ERR_INVALID_ARG, "handle, idx or counts is NULL");
    if (h->last_n < 0) return fail(SFFN_ERR_NOT_READY, "no forward has run");
    DeviceGuard g(h->cfg.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    SFFN_CUDA(cudaStreamSynchronize(h->last_stream), "stream synchronize");
    int rc = sffn_check_status(h);
    if (rc) return rc;
    const Plan& P = h->plan;
    const int n = h->last_n, F = h->cfg.d_ff;
    std::vector<int> seg(P.g1), lidx(F);
    std::vector<uint32_t> mask((size_t)F * P.mw);
    if (h->last_tc) {
        // the tensor-core path keeps the gate's decisions, not lists: z (threshold,
        // the same fp32 comparison the kernels make) or the top-K mask
        for (int t = 0; t < n; ++t) counts[t] = 0;
        std::vector<uint8_t> any(F, 0);
        if (h->last_topk) {
            std::vector<uint8_t> selv((size_t)n * F);
            SFFN_CUDA(cudaMemcpy(selv.data(), h->sel, selv.size(), cudaMemcpyDeviceToHost), "mask copy");
            for (int t = 0; t < n; ++t)
                for (int k = 0; k < F; ++k)
                    if (selv[(size_t)t * F + k]) {
                        idx[(size_t)t * F + counts[t]++] = k;
                        any[k] = 1;
                    }
        } else {
            // the gate kernel's own per-token selection bits
            const int W = h->selw;
            std::vector<uint32_t> bits((size_t)n * W);
            SFFN_CUDA(cudaMemcpy(bits.data(), h->selbits, bits.size() * 4, cudaMemcpyDeviceToHost), "selection copy");
            for (int t = 0; t < n; ++t)
                for (int k = 0; k < F; ++k)
                    if ((bits[(size_t)t * W + (k >> 5)] >> (k & 31)) & 1u) {
                        idx[(size_t)t * F + counts[t]++] = k;
                        any[k] = 1;
                    }
            // bits past d_ff in the last word must be clear
            if (F & 31)
                for (int t = 0; t < n; ++t)
                    if (bits[(size_t)t * W + W - 1] >> (F & 31))
                        return fail(SFFN_ERR_DEVICE_CHECK, "selection bit past d_ff for token %d", t);
        }
        int uni = 0;
        for (int k = 0; k < F; ++k) uni += any[k];
        if (union_size) *union_size = uni;
        return SFFN_OK;
    }
    SFFN_CUDA(cudaMemcpy(seg.data(), h->seg_count, seg.size() * 4, cudaMemcpyDeviceToHost), "list copy");
    SFFN_CUDA(cudaMemcpy(lidx.data(), h->lst_idx, lidx.size() * 4, cudaMemcpyDeviceToHost), "list copy");
    SFFN_CUDA(cudaMemcpy(mask.data(), h->lst_mask, mask.size() * 4, cudaMemcpyDeviceToHost), "list copy");
    for (int t = 0; t < n; ++t) counts[t] = 0;
    int uni = 0;
    for (int b = 0; b < P.g1; ++b) {
        if (seg[b] < 0 || seg[b] > P.cpb || (long long)b * P.cpb + seg[b] > F)
            return fail(SFFN_ERR_DEVICE_CHECK, "segment %d count %d", b, seg[b]);
        for (int i = 0; i < seg[b]; ++i) {
            const int k = lidx[(size_t)b * P.cpb + i];
            if (k < b * P.cpb || k >= F) return fail(SFFN_ERR_DEVICE_CHECK, "listed channel %d out of range", k);
            bool any = false;
            for (int t = 0; t < n; ++t)
                if ((mask[(size_t)k * P.mw + (t >> 5)] >> (t & 31)) & 1u) {
                    idx[(size_t)t * F + counts[t]++] = k;
                    any = true;
                }
            uni += any;
        }
    }
    if (union_size) *union_size = uni;
    return SFFN_OK;
}

int sffn_get_union(sffn_handle h, uint32_t* bits, int nwords) {
    if (!h || !bits) return fail(SFFN_ERR_INVALID_ARG, "handle or bits is NULL");
    const int W = (h->cfg.d_ff + 31) / 32;
    if (nwords < W) return fail(SFFN_ERR_INVALID_ARG, "nwords=%d < ceil(d_ff / 32)=%d", nwords, W);
    if (h->last_n < 0) return fail(SFFN_ERR_NOT_READY, "no forward has run");
    if (!h->last_tc) return fail(SFFN_ERR_UNSUPPORTED, "the last forward did not take the tensor-core path");
    DeviceGuard g(h->cfg.device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    SFFN_CUDA(cudaStreamSynchronize(h->last_stream), "stream synchronize");
    const int rc = sffn_check_status(h);
    if (rc) return rc;
    SFFN_CUDA(cudaMemcpy(bits, h->ubits, (size_t)W * 4, cudaMemcpyDeviceToHost), "union copy");
    for (int w = W; w < nwords; ++w) bits[w] = 0u;
    return SFFN_OK;
}

int sffn_debug_inject(sffn_handle h, int what, long long arg) {
    if (!h) return fail(SFFN_ERR_INVALID_ARG, "handle is NULL");
    switch (what) {
        case SFFN_INJECT_WAIT_TIMEOUT:
            if (arg < 1000 || arg > 2000000000LL)
                return fail(SFFN_ERR_INVALID_ARG, "wait limit %lld ns outside [1 us, 2 s]", arg);
            h->inj_wait_ns = (unsigned long long)arg;
            return SFFN_OK;
        case SFFN_INJECT_BAD_LIST_ENTRY:
            h->inj_bad_index = true;
            return SFFN_OK;
        default:
            return fail(SFFN_ERR_INVALID_ARG, "unknown injection %d", what);
    }
}

int sffn_set_hot(sffn_handle h, const int32_t* channels, int count) {
    if (!h || count < 0 || (count > 0 && !channels)) return fail(SFFN_ERR_INVALID_ARG, "bad hot channel list");
    const int d_ff = h->cfg.d_ff;
    std::vector<uint32_t> bits(((size_t)d_ff + 31) / 32, 0u);
    for (int i = 0; i < count; ++i) {
        if (channels[i] < 0 || channels[i] >= d_ff) return fail(SFFN_ERR_INVALID_ARG, "hot channel out of range");
        bits[(size_t)channels[i] >> 5] |= 1u << (channels[i] & 31);
    }
    DeviceGuard g(h->cfg.device);
    if (count == 0 && !h->hot) return SFFN_OK;
    // The buffer is never freed before the handle, so a graph captured with
    // an earlier set keeps a valid (all-clear after a clear) bitmap.
    if (!h->hot) {
        void* p = nullptr;
        if (cudaMalloc(&p, bits.size() * sizeof(uint32_t)) != cudaSuccess) {
            cudaGetLastError();
            return fail(SFFN_ERR_OOM, "hot set allocation");
        }
        h->hot = static_cast<uint32_t*>(p);
    }
    // earlier forwards may still read the old set
    SFFN_CUDA(cudaDeviceSynchronize(), "hot set update");
    SFFN_CUDA(cudaMemcpy(h->hot, bits.data(), bits.size() * sizeof(uint32_t), cudaMemcpyHostToDevice), "hot set copy");
    h->hot_on = count > 0;
    return SFFN_OK;
}

int sffn_set_stage_events(sffn_handle h, void* const* events, int n_events) {
    if (!h || n_events < 0 || (n_events > 0 && !events)) return fail(SFFN_ERR_INVALID_ARG, "bad events");
    h->events.clear();
    for (int i = 0; i < n_events; ++i) h->events.push_back(static_cast<cudaEvent_t>(events[i]));
    return SFFN_OK;
}

int sffn_last_launches(sffn_handle h, int32_t* launches) {
    if (!h || !launches) return fail(SFFN_ERR_INVALID_ARG, "handle or launches is NULL");
    *launches = h->last_launches;
    return SFFN_OK;
}

const char* sffn_last_kernel_name(sffn_handle h, int i) {
    if (!h || i < 0 || i >= h->last_launches || i >= 64 || !h->last_names[i]) return "";
    return h->last_names[i];
}

int sffn_destroy(sffn_handle h) {
    if (!h) return SFFN_OK;
    {
        DeviceGuard g(h->cfg.device);
        free_weights(h);
        if (h->ws) cudaFree(h->ws);
        if (h->hot) cudaFree(h->hot);
        if (h->hstat) cudaFreeHost(h->hstat);
    }
    delete h;
    return SFFN_OK;
}

}  // extern "C"
