// Sparse forward that allocates nothing (sffn_forward_noalloc).
//
// For callers that may not call cudaMalloc once they are running: a host
// runtime that owns every byte of device memory through its own pool, a
// process that must not allocate after start-up because an allocation can
// synchronise the device and stall latency-critical work, or code that runs
// where the CUDA allocator is off limits.  Such a caller hands over its weights
// (already in the channel-major layout the kernels read), x and the output; the
// scratch the kernels need lives in one file-scope device array, reserved when
// the library is loaded and held by every GPU that loads it until the process
// exits.
//
// The kernels are the library's own (streaming gate with threshold select and
// up projection, then the gathered down projection); only where their scratch
// comes from differs.  Dense gate and threshold selection only.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "sffn.h"

namespace sffn {
namespace {

// Limits of the scratch array.
constexpr int kNaMaxD = 8192;
constexpr int kNaMaxDff = 32768;
constexpr int kNaMaxTokens = 8;
constexpr int kNaMaxSms = 192;
constexpr int kNaMaxSlices = kNaMaxD / 512;

constexpr size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Scratch layout (bytes), fixed by the limits above.
constexpr size_t kOffIdx = 0;
constexpr size_t kOffH = kOffIdx + align256((size_t)kNaMaxDff * 4);
constexpr size_t kOffMask = kOffH + align256((size_t)kNaMaxDff * kNaMaxTokens * 4);
constexpr size_t kOffSeg = kOffMask + align256((size_t)kNaMaxDff * 4);
constexpr size_t kOffPart = kOffSeg + align256((size_t)2 * kNaMaxSms * 4);
// down partials: chunks * n * d floats with chunks * slices <= SMs, slices = ceil(d / 512)
constexpr size_t kOffTickets = kOffPart + align256((size_t)kNaMaxSms * 512 * kNaMaxTokens * 4);
constexpr size_t kOffStatus = kOffTickets + align256((size_t)kNaMaxSlices * 4);
constexpr size_t kScratchBytes = kOffStatus + 256;   // about 3.9 MiB

// The scratch itself.  In host code this name is only a stand-in for the
// device array: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

thread_local char g_na_err[256] = "";
std::mutex g_na_mutex;
void* g_na_ptr[64] = {};
int g_na_sms[64] = {};

int na_fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_na_err, sizeof g_na_err, fmt, ap);
    va_end(ap);
    fprintf(stderr, "sffn_forward_noalloc: %s\n", g_na_err);
    return code;
}

// Once per device, with that device current: the array's device address and
// the SM count.  Later calls reuse both.
int na_setup(int dev, void** ptr, int* sms) {
    std::lock_guard<std::mutex> lock(g_na_mutex);
    if (!g_na_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) return na_fail(SFFN_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess || n <= 0) return na_fail(SFFN_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
        g_na_sms[dev] = n < kNaMaxSms ? n : kNaMaxSms;
        g_na_ptr[dev] = p;
    }
    *ptr = g_na_ptr[dev];
    *sms = g_na_sms[dev];
    return SFFN_OK;
}

}  // namespace
}  // namespace sffn

using namespace sffn;

extern "C" int sffn_forward_noalloc(const void* w_gate_cm, const void* w_up_cm, const void* w_down, int d,
                                    int d_ff, int wdtype, const void* x, int n_tokens, float tau, void* out,
                                    void* stream) {
    if (d <= 0 || d % 8 || d > kNaMaxD)
        return na_fail(SFFN_ERR_INVALID_ARG, "d=%d must be a multiple of 8 in [8, %d]", d, kNaMaxD);
    if (d_ff <= 0 || d_ff > kNaMaxDff)
        return na_fail(SFFN_ERR_INVALID_ARG, "d_ff=%d must be in [1, %d]", d_ff, kNaMaxDff);
    if (n_tokens < 0 || n_tokens > kNaMaxTokens)
        return na_fail(SFFN_ERR_INVALID_ARG, "n_tokens=%d must be in [0, %d]", n_tokens, kNaMaxTokens);
    if (wdtype != SFFN_BF16 && wdtype != SFFN_F32) return na_fail(SFFN_ERR_INVALID_ARG, "unknown wdtype %d", wdtype);
    if (std::isnan(tau) || (std::isinf(tau) && tau < 0))
        return na_fail(SFFN_ERR_INVALID_ARG, "tau must be a number or +inf");
    if (n_tokens == 0) return SFFN_OK;
    for (const void* p : {w_gate_cm, w_up_cm, w_down, x, (const void*)out})
        if (!p || (reinterpret_cast<uintptr_t>(p) & 15u))
            return na_fail(SFFN_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return na_fail(SFFN_ERR_CUDA, "cudaGetDevice failed");
    void* base = nullptr;
    int sms = 0;
    int rc = na_setup(dev, &base, &sms);
    if (rc) return rc;
    char* b = static_cast<char*>(base);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Plan: one gate CTA per SM; down chunks so that slices x chunks ~ SMs.
    const int cpb = (d_ff + sms - 1) / sms;
    const int g1 = (d_ff + cpb - 1) / cpb;
    const int slices = (d + down_slice_cols(wdtype) - 1) / down_slice_cols(wdtype);
    int chunks = sms / slices;
    if (chunks < 1) chunks = 1;
    if (chunks > g1) chunks = g1;
    const int nt = n_tokens <= 1 ? 1 : n_tokens <= 2 ? 2 : n_tokens <= 4 ? 4 : 8;
    int gnt = nt, sb = 0, nb = 0;
    size_t gsmem = 0;
    while (!gate_stream_geometry(gnt, d, 0, kGateDense, cpb, 1, &sb, &nb, &gsmem) && gnt > 1) gnt /= 2;
    if (!sb) return na_fail(SFFN_ERR_UNSUPPORTED, "shape does not fit shared memory");

    // The ticket counters must start at zero: clear them.  The status word is
    // left alone: it keeps every failure until sffn_noalloc_check_status reads it.
    e = cudaMemsetAsync(b + kOffTickets, 0, kOffStatus - kOffTickets, s);
    if (e != cudaSuccess) return na_fail(SFFN_ERR_CUDA, "clearing scratch: %s", cudaGetErrorString(e));

    GateParams gp{};
    gp.x = x; gp.n = n_tokens; gp.d = d; gp.d_ff = d_ff; gp.r = 0;
    gp.wg = w_gate_cm; gp.wup = w_up_cm; gp.wdn = w_down;
    gp.out = kOutSelectUp; gp.force_all = 0; gp.tau = tau;
    gp.cpb = cpb; gp.mw = 1;
    gp.lst_idx = reinterpret_cast<int*>(b + kOffIdx);
    gp.lst_h = reinterpret_cast<float*>(b + kOffH);
    gp.lst_mask = reinterpret_cast<uint32_t*>(b + kOffMask);
    gp.seg_count = reinterpret_cast<int*>(b + kOffSeg);
    gp.sb = sb; gp.nb = nb;
    gp.status = reinterpret_cast<int*>(b + kOffStatus);
    e = launch_gate_stream(wdtype, gp, gnt, kGateDense, g1, gsmem, s, true);
    if (e != cudaSuccess) return na_fail(SFFN_ERR_CUDA, "gate launch: %s", cudaGetErrorString(e));

    DownParams dp{};
    dp.wdn = w_down; dp.n = n_tokens; dp.d = d; dp.d_ff = d_ff;
    dp.seg_count = gp.seg_count; dp.g1 = g1; dp.cpb = cpb;
    dp.lst_idx = gp.lst_idx; dp.lst_h = gp.lst_h;
    dp.part = reinterpret_cast<float*>(b + kOffPart);
    dp.tickets = reinterpret_cast<unsigned*>(b + kOffTickets);
    dp.y = out; dp.chunks = chunks; dp.status = gp.status;
    const int nseg = (g1 + chunks - 1) / chunks;
    e = launch_down(wdtype, dp, nt, slices, down_smem_bytes(wdtype, nt, nseg, cpb), s, true);
    if (e != cudaSuccess) return na_fail(SFFN_ERR_CUDA, "down launch: %s", cudaGetErrorString(e));
    return SFFN_OK;
}

// Read, then clear, the status word in this device's scratch.
extern "C" int sffn_noalloc_check_status(void) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return na_fail(SFFN_ERR_CUDA, "cudaGetDevice failed");
    void* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_na_mutex);
        base = g_na_ptr[dev];
    }
    if (!base) return SFFN_OK;                 // no call has run on this device
    int* st = reinterpret_cast<int*>(static_cast<char*>(base) + kOffStatus);
    int v = 0;
    e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&v, st, sizeof v, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v) e = cudaMemset(st, 0, sizeof v);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return na_fail(SFFN_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v & kStatusBounds) return na_fail(SFFN_ERR_DEVICE_CHECK, "a bounds check failed (status 0x%x)", v);
    if (v & kStatusWaitTimeout) return na_fail(SFFN_ERR_TIMEOUT, "a bounded wait timed out (status 0x%x)", v);
    if (v) return na_fail(SFFN_ERR_DEVICE_CHECK, "status word 0x%x", v);
    return SFFN_OK;
}
