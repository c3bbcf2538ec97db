// Batched path on the 5th-generation tensor cores (tcgen05).
//
// With several tokens per step the gate and the gathered up and down passes
// are dense contractions (a token batch against weight rows), so they run as
// one tcgen05 GEMM kernel with three epilogues:
//
//   gate   Z^T[rows x n] = W[rows x K] . X^T      A = weight rows (K-major),
//                                                 B = x rows (K-major)
//   up     H^T[U x n]    = W_up[union rows] . X^T, times the gate activation
//   down   Y^T[d x n]    = W_down[union rows]^T . H^T
//                                                 A = W_down rows read as an
//                                                 MN-major operand, B = H rows
//
// "Model Casting and Low-Parameter Gating" (abstract): gate first, then only
// the active channels' rows of the other two matrices.  "Mixture-of-Channels"
// (section "Dentro MoC"): rows of the union of the batch's selected channels
// are loaded once and shared by the tokens that selected them; a token that
// did not select a channel gets a zero activation for it.
//
// Kernel structure (one CTA per SM, 288 threads):
//   warps 0-3  producers: cp.async 16-byte copies of the A and B tiles of each
//              64-wide k-block straight into the 128-byte-swizzled shared
//              memory layout the MMA reads (rows gathered through the union
//              list where needed), a ring of up to 8 stages on mbarriers;
//   warp 8     one thread issues tcgen05.mma (M = 128, N = token columns,
//              K = 16 per instruction, bf16 in, fp32 accumulate in tensor
//              memory) and tcgen05.commit to release stages and accumulators;
//   warps 4-7  epilogue: tcgen05.ld of the accumulator (each warp its 32 TMEM
//              lanes), the mode's epilogue, stores.
// Work is split stream-K: the (tile, k-block) iterations are cut into one
// contiguous range per CTA, so every SM streams the same number of weight
// bytes.  A tile cut between CTAs is summed in a fixed order (by CTA index)
// by the CTA that completes it last (ticket), so results are deterministic.
//
// fp32 intermediates that feed a later MMA (LoPA's u = x A, and h) are passed
// as two bf16 rows, hi = bf16(v) and lo = bf16(v - hi); the MMA multiplies both
// and the epilogue adds the two columns, which keeps about 16 significant bits.
#include "common.cuh"

namespace sffn {
namespace {

constexpr int kBM = 128;            // accumulator rows (MMA M)
constexpr int kBK = 64;             // k-block: 64 bf16 = one 128-byte swizzle row
constexpr int kProd = 4;            // producer warps
constexpr int kEpi = 4;             // epilogue warps
constexpr int kMmaWarp = kProd + kEpi;
constexpr int kTcThreads = (kProd + kEpi + 1) * 32;
constexpr uint32_t kTileA = kBM * kBK * 2;   // 16 KB
constexpr int kMaxStages = 8;

struct TcShared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int reducer;
    int rows[kBM];          // up: union rows of the current tile
};

// ---- tcgen05 / cp.async primitives -------------------------------------------

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
                 "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulator).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}
// 16 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// One thread waits (bounded) for the phase with `parity`.
__device__ __forceinline__ bool mbar_wait_one(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}
// 16-byte global -> shared copy; src_bytes 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t src_bytes, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src),
                 "r"(src_bytes), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, version 1 (sm_100).
// K-major: 8-row groups `sbo` bytes apart (rows 128 B apart inside a group).
// MN-major: 64-element MN blocks `lbo` bytes apart, 8-k groups `sbo` apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;        // descriptor version for sm_100
    d |= (uint64_t)2 << 61;        // SWIZZLE_128B
    return d;
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 128, N = n.
__device__ __forceinline__ uint32_t mma_idesc(int n, int a_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kBM >> 4) << 24);
}
// Byte offset of 16-byte chunk c (0..7) of row r in a K-major 128B-swizzled
// tile whose 8-row groups are 1024 B apart.
__device__ __forceinline__ uint32_t kmaj_off(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void set_status(int* st, int bits) {
    if (st) atomicOr(st, bits);
}

// The CTA c whose range [floor(c I/C), floor((c+1) I/C)) holds iteration i
// (C <= I, so no range is empty).
__device__ __forceinline__ int cta_of(long long i, long long I, int C) {
    return (int)(((i + 1) * C - 1) / I);
}

struct Seg {
    int t, kb0, kb1;
};

struct Problem {
    int T, KB, U;
    int MT;                 // 128-row accumulator tiles per work tile (down: MN-major, several)
    int C;                  // CTAs that take work: min(grid, I), so none has an empty range
    long long I, it0, it1;
};

__device__ __forceinline__ Problem make_problem(const TcParams& p) {
    Problem q;
    q.U = p.u_count ? min(max(*p.u_count, 0), p.u_cap) : 0;
    q.MT = p.mode == kTcDown ? p.mt : 1;
    const int kstep = kBK * p.ks;                     // contraction per iteration
    if (p.mode == kTcUp) {
        q.T = (q.U + kBM - 1) / kBM;
        q.KB = (p.k_total + kstep - 1) / kstep;
    } else if (p.mode == kTcDown) {
        q.T = (p.m_total + kBM * q.MT - 1) / (kBM * q.MT);
        q.KB = (q.U + kstep - 1) / kstep;
    } else {
        q.T = (p.m_total + kBM - 1) / kBM;
        q.KB = (p.k_total + kstep - 1) / kstep;
    }
    q.I = (long long)q.T * q.KB;
    q.C = (int)min((long long)gridDim.x, q.I);
    if ((int)blockIdx.x < q.C) {
        q.it0 = q.I * blockIdx.x / q.C;
        q.it1 = q.I * (blockIdx.x + 1) / q.C;
    } else {
        q.it0 = q.it1 = 0;
    }
    return q;
}

__device__ __forceinline__ bool next_seg(const Problem& q, long long& it, Seg& s) {
    if (it >= q.it1) return false;
    s.t = (int)(it / q.KB);
    s.kb0 = (int)(it % q.KB);
    s.kb1 = (int)min((long long)q.KB, s.kb0 + (q.it1 - it));
    it += s.kb1 - s.kb0;
    return true;
}

// Stage layout: A sub-tiles of 16 KB (gate/up: one per 64-wide k-block of the
// iteration; down: one per 128-row accumulator tile), then B sub-tiles of
// nb x 128 B (one per 64-wide k-block).
__device__ __forceinline__ int a_subtiles(const TcParams& p) { return p.mode == kTcDown ? p.mt : p.ks; }

// ---- producer: A and B tiles of one iteration into stage memory ---------------

template <int LAG>
__device__ void run_producer(const TcParams& p, const Problem& q, unsigned char* stages, uint32_t stage_bytes,
                             TcShared* sh) {
    const int tid = threadIdx.x;                      // 0..127
    const int w = tid >> 5, l = tid & 31;
    const uint64_t pol_w = l2_evict_first(), pol_b = l2_evict_last();
    const bf16* A = static_cast<const bf16*>(p.a);
    const bf16* B = static_cast<const bf16*>(p.b);
    const int S = p.stages;
    const int KS = p.ks;
    const int CPR = KS * 8;                           // 16-byte chunks of a K-major row per iteration
    const int RPI = 32 / CPR;                         // rows per warp instruction (4, 2 or 1)
    const int rsub = l / CPR, chunk = l % CPR;
    const int kstep = kBK * KS;
    const uint32_t b_off = (uint32_t)a_subtiles(p) * kTileA;
    long long it = q.it0;
    long long g = 0;                                  // iterations issued by this CTA
    Seg s;
    bool ok = true;
    while (ok && next_seg(q, it, s)) {
        const int m0 = s.t * kBM * q.MT;
        if (p.mode == kTcUp) {
            // the tile's 128 union rows, shared by the producer warps
            named_sync(2, kProd * 32);
            const int m = m0 + tid;
            sh->rows[tid] = m < q.U ? __ldg(p.a_rows + m) : -1;
            named_sync(2, kProd * 32);
        }
        // down: the union rows of iteration kb (k-rows w + 4 j), fetched one iteration ahead
        int rcur[16], rnxt[16];
        if (p.mode == kTcDown) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int pos = s.kb0 * kBK + w + 4 * j;
                rcur[j] = pos < q.U ? __ldg(p.a_rows + pos) : -1;
            }
        }
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++g) {
            if (p.mode == kTcDown) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int pos = (kb + 1) * kBK + w + 4 * j;
                    rnxt[j] = (kb + 1 < s.kb1 && pos < q.U) ? __ldg(p.a_rows + pos) : -1;
                }
            }
            const int st = (int)(g % S);
            const uint32_t use = (uint32_t)(g / S);
            if (!mbar_wait_warp(&sh->empty[st], (use & 1u) ^ 1u)) {
                sh->abort = 1;
                set_status(p.status, kStatusWaitTimeout);
                ok = false;
                break;
            }
            const uint32_t sA = smem_addr(stages + (size_t)st * stage_bytes);
            const uint32_t sB = sA + b_off;
            const int k0 = kb * kstep;
            if (p.mode != kTcDown) {
                // K-major A: row r, chunk `chunk` of its KS*128 contiguous bytes
                const int sub = chunk >> 3, c = chunk & 7;
                const int k = k0 + chunk * 8;
                for (int r = w * RPI + rsub; r < kBM; r += 4 * RPI) {
                    long long row;
                    bool v;
                    if (p.mode == kTcUp) {
                        row = sh->rows[r];
                        v = row >= 0;
                    } else {
                        row = m0 + r;
                        v = row < p.m_total;
                    }
                    v = v && k < p.k_total;
                    const bf16* src = v ? A + row * p.lda + k : A;
                    cp16(sA + sub * kTileA + kmaj_off(r, c), src, v ? 16u : 0u, pol_w);
                }
            } else {
                // MN-major A: k-row kr holds W_down[list[kb*64+kr]][m0 .. m0 + 128 MT); 16 MT chunks
                const int cpr = q.MT * 16;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int kr = w + 4 * j;
                    for (int qc = l; qc < cpr; qc += 32) {
                        const int mt = qc >> 4, c16 = qc & 15;
                        const int col = m0 + qc * 8;
                        const bool v = rcur[j] >= 0 && col < p.m_total;
                        const bf16* src = v ? A + (long long)rcur[j] * p.lda + col : A;
                        const uint32_t off = (uint32_t)(mt * kTileA + (c16 >> 3) * 8192 + (kr >> 3) * 1024 +
                                                        (kr & 7) * 128 + (((c16 & 7) ^ (kr & 7)) << 4));
                        cp16(sA + off, src, v ? 16u : 0u, pol_w);
                    }
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) rcur[j] = rnxt[j];
            }
            // B: nb rows, KS*128 contiguous bytes each
            {
                const int sub = chunk >> 3, c = chunk & 7;
                const int k = k0 + chunk * 8;
                for (int r = w * RPI + rsub; r < p.nb; r += 4 * RPI) {
                    const bool v = r < p.b_rows && k < p.b_cols;
                    const bf16* src = v ? B + (long long)r * p.ldb + k : B;
                    cp16(sB + sub * (uint32_t)p.nb * 128u + kmaj_off(r, c), src, v ? 16u : 0u, pol_b);
                }
            }
            cp_commit();
            if (g >= LAG) {
                cp_wait<LAG>();
                fence_proxy_async();
                mbar_arrive(&sh->full[(int)((g - LAG) % S)]);
            }
        }
    }
    // every copy lands before the CTA can retire; arrive for the stages not yet signalled
    cp_wait<0>();
    fence_proxy_async();
    if (ok)
        for (long long h = (g >= LAG ? g - LAG : 0); h < g; ++h) mbar_arrive(&sh->full[(int)(h % S)]);
}

// ---- MMA issuer --------------------------------------------------------------

__device__ void run_mma(const TcParams& p, const Problem& q, unsigned char* stages, uint32_t stage_bytes,
                        TcShared* sh, uint32_t tmem) {
    const int S = p.stages;
    const bool down = p.mode == kTcDown;
    const uint32_t idesc = mma_idesc(p.nb, down ? 1 : 0);
    const uint32_t b_off = (uint32_t)a_subtiles(p) * kTileA;
    const int acc_cols = q.MT * p.nb;
    long long it = q.it0, g = 0;
    int segi = 0;
    Seg s;
    bool ok = true;
    while (ok && next_seg(q, it, s)) {
        const int acc = segi & 1;
        const uint32_t use = (uint32_t)(segi >> 1);
        if (!mbar_wait_one(&sh->tempty[acc], (use & 1u) ^ 1u)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * acc_cols);
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++g) {
            const int st = (int)(g % S);
            if (!mbar_wait_one(&sh->full[st], (uint32_t)((g / S) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sA = smem_addr(stages + (size_t)st * stage_bytes);
            const uint32_t sB = sA + b_off;
            if (down) {
                for (int mt = 0; mt < q.MT; ++mt)
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma(d_tmem + mt * p.nb, sw128_desc(sA + mt * kTileA + kk * 2048, 8192, 1024),
                               sw128_desc(sB + kk * 32, 16, 1024), idesc, (kb > s.kb0 || kk > 0) ? 1u : 0u);
            } else {
                for (int sub = 0; sub < p.ks; ++sub)
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc_mma(d_tmem, sw128_desc(sA + sub * kTileA + kk * 32, 16, 1024),
                               sw128_desc(sB + sub * p.nb * 128 + kk * 32, 16, 1024), idesc,
                               (kb > s.kb0 || sub > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&sh->empty[st]);
        }
        if (!ok) break;
        tc_commit(&sh->tfull[acc]);
        ++segi;
    }
    if (!ok) {
        sh->abort = 1;
        set_status(p.status, kStatusWaitTimeout);
    }
    // all issued MMAs complete before the accumulators are released
    tc_commit(&sh->drain);
    mbar_wait_one(&sh->drain, 0);
}

// ---- epilogue ----------------------------------------------------------------

// Final values v[0..15] of columns c0..c0+15 (combined hi+lo when paired) for
// output row m.  `act` collects the gate's activity flag.
__device__ __forceinline__ void emit16(const TcParams& p, const Problem& q, int m, int c0, const float* v,
                                       bool& act) {
    if (p.mode == kTcGateZ) {
        if (m >= p.m_total) return;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int tok = c0 + i;
            if (tok < p.n) {
                p.z[(long long)tok * p.ldz + m] = v[i];
                act |= v[i] > p.tau;
            }
        }
    } else if (p.mode == kTcGateSplit) {
        if (m >= p.m_total) return;
        bf16* o = static_cast<bf16*>(p.out);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int tok = c0 + i;
            const bf16 hi = __float2bfloat16_rn(v[i]);
            const bf16 lo = __float2bfloat16_rn(v[i] - __bfloat162float(hi));
            o[(long long)tok * p.ldo + m] = hi;
            o[(long long)(p.npad + tok) * p.ldo + m] = lo;
        }
    } else if (p.mode == kTcUp) {
        bf16* o = static_cast<bf16*>(p.out);
        const int ch = m < q.U ? __ldg(p.a_rows + m) : -1;
        float gv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int tok = c0 + i;
            gv[i] = 0.f;
            if (ch >= 0 && tok < p.n) {
                const long long zi = (long long)tok * p.ldsel + ch;
                gv[i] = p.topk ? p.gsel[zi] : fmaxf(p.zsel[zi] - p.tau, 0.f);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int tok = c0 + i;
            const float h = gv[i] * v[i];
            const bf16 hi = __float2bfloat16_rn(h);
            o[(long long)tok * p.ldo + m] = hi;
            if (p.h_pairs) o[(long long)(p.npad + tok) * p.ldo + m] = __float2bfloat16_rn(h - __bfloat162float(hi));
        }
    } else {  // down
        if (m >= p.m_total) return;
        bf16* o = static_cast<bf16*>(p.out);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int tok = c0 + i;
            if (tok < p.n) o[(long long)tok * p.ldo + m] = __float2bfloat16_rn(v[i]);
        }
    }
}

__device__ void run_epilogue(const TcParams& p, const Problem& q, TcShared* sh, uint32_t tmem) {
    const int ew = (threadIdx.x >> 5) & 3;            // TMEM lane quarter of this warp
    const int lane = threadIdx.x & 31;
    const int row = ew * 32 + lane;
    const int etid = threadIdx.x - kProd * 32;        // 0..127
    const int cols = p.paired ? p.npad : p.nb;        // final columns
    const int C = q.C;
    const int acc_cols = q.MT * p.nb;
    const size_t slot_floats = (size_t)acc_cols * kBM;
    long long it = q.it0;
    int segi = 0;
    Seg s;
    while (next_seg(q, it, s)) {
        const int acc = segi & 1;
        const uint32_t use = (uint32_t)(segi >> 1);
        ++segi;
        if (!mbar_wait_warp(&sh->tfull[acc], use & 1u)) {
            sh->abort = 1;
            set_status(p.status, kStatusWaitTimeout);
            return;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * acc_cols);
        const bool whole = s.kb0 == 0 && s.kb1 == q.KB;
        const int mbase = s.t * kBM * q.MT + row;
        bool act = false;
        if (whole) {
            for (int mt = 0; mt < q.MT; ++mt)
                for (int c0 = 0; c0 < cols; c0 += 16) {
                    float v[16];
                    tmem_ld16(taddr + mt * p.nb + c0, v);
                    if (p.paired) {
                        float x[16];
                        tmem_ld16(taddr + mt * p.nb + p.npad + c0, x);
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] += x[i];
                    }
                    emit16(p, q, mbase + mt * kBM, c0, v, act);
                }
            tc_fence_before();
            mbar_arrive(&sh->tempty[acc]);
        } else {
            // partial tile: park it, the CTA completing the tile sums all parts in CTA order
            const int c_first = cta_of((long long)s.t * q.KB, q.I, C);
            const int slot = c_first == (int)blockIdx.x ? 0 : 1;
            float* mine = p.part + ((size_t)blockIdx.x * 2 + slot) * slot_floats;
            for (int c0 = 0; c0 < acc_cols; c0 += 16) {
                float v[16];
                tmem_ld16(taddr + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) mine[(size_t)(c0 + i) * kBM + row] = v[i];
            }
            tc_fence_before();
            mbar_arrive(&sh->tempty[acc]);
            __threadfence();
            named_sync(1, kEpi * 32);
            const int c_last = cta_of((long long)(s.t + 1) * q.KB - 1, q.I, C);
            if (etid == 0) {
                const unsigned done = atomicAdd(p.tickets + s.t, 1u);
                sh->reducer = done == (unsigned)(c_last - c_first);
                if (sh->reducer) p.tickets[s.t] = 0;   // every part has arrived: reset for the next launch
            }
            named_sync(1, kEpi * 32);
            const bool red = sh->reducer != 0;
            named_sync(1, kEpi * 32);
            if (!red) continue;
            __threadfence();
            for (int mt = 0; mt < q.MT; ++mt)
                for (int c0 = 0; c0 < cols; c0 += 16) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.f;
                    for (int c = c_first; c <= c_last; ++c) {
                        const float* pp = p.part + ((size_t)c * 2 + (c == c_first ? 0 : 1)) * slot_floats +
                                          (size_t)mt * p.nb * kBM;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float x = __ldcg(pp + (size_t)(c0 + i) * kBM + row);
                            if (p.paired) x += __ldcg(pp + (size_t)(p.npad + c0 + i) * kBM + row);
                            v[i] += x;
                        }
                    }
                    emit16(p, q, mbase + mt * kBM, c0, v, act);
                }
        }
        if (p.mode == kTcGateZ && p.ubits) {
            // union bitmap words of this tile: one word per warp (32 channels)
            const unsigned bits = __ballot_sync(0xffffffffu, act && !p.topk && mbase < p.m_total);
            if (lane == 0) p.ubits[(s.t * kBM + ew * 32) >> 5] = bits;
        }
    }
}

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_gemm(const TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* stages = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                             ~static_cast<uintptr_t>(1023));
    const uint32_t stage_bytes = (uint32_t)a_subtiles(p) * kTileA + (uint32_t)(p.ks * p.nb) * 128u;
    TcShared* sh = reinterpret_cast<TcShared*>(stages + (size_t)p.stages * stage_bytes);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) {
            mbar_init(&sh->full[i], kProd * 32);
            mbar_init(&sh->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->tfull[i], 1);
            mbar_init(&sh->tempty[i], kEpi * 32);
        }
        mbar_init(&sh->drain, 1);
        sh->abort = 0;
        sh->reducer = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&sh->tmem_base, p.tmem_cols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    griddep_launch_dependents();
    griddep_wait();
    const Problem q = make_problem(p);

    if (warp < kProd) {
        if (p.stages >= 8) run_producer<6>(p, q, stages, stage_bytes, sh);
        else if (p.stages >= 6) run_producer<4>(p, q, stages, stage_bytes, sh);
        else run_producer<2>(p, q, stages, stage_bytes, sh);
    } else if (warp < kProd + kEpi) {
        run_epilogue(p, q, sh, tmem);
    } else if ((threadIdx.x & 31) == 0) {
        run_mma(p, q, stages, stage_bytes, sh, tmem);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, p.tmem_cols);
}

// ---- union list ----------------------------------------------------------------
// Ordered list of the channels any token selected (bit k of the bitmap), the
// per-channel token masks, and the union size.

constexpr int kUnionThreads = 1024;

__global__ void __launch_bounds__(kUnionThreads) k_union(const UnionParams p) {
    __shared__ int sh[40];
    __shared__ int s_red[32];
    griddep_launch_dependents();
    griddep_wait();
    const int base = blockIdx.x * kUnionThreads;
    const int words_before = base >> 5;
    const int nwords = (p.d_ff + 31) >> 5;
    // channels listed before this block: popcount of the bitmap words before it
    int before = 0, total = 0;
    if (p.force_all) {
        before = base;
        total = p.d_ff;
    } else {
        int a = 0, b = 0;
        for (int w = threadIdx.x; w < nwords; w += kUnionThreads) {
            const uint32_t bits = p.ubits[w];
            const int c = __popc(w == nwords - 1 && (p.d_ff & 31) ? bits & ((1u << (p.d_ff & 31)) - 1u) : bits);
            b += c;
            if (w < words_before) a += c;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, o);
            b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = a;
        __syncthreads();
        if (threadIdx.x < 32) {
            int x = s_red[threadIdx.x];
#pragma unroll
            for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (threadIdx.x == 0) s_red[0] = x;
        }
        __syncthreads();
        before = s_red[0];
        __syncthreads();
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = b;
        __syncthreads();
        if (threadIdx.x < 32) {
            int x = s_red[threadIdx.x];
#pragma unroll
            for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (threadIdx.x == 0) s_red[1] = x;
        }
        __syncthreads();
        total = s_red[1];
    }
    const int k = base + threadIdx.x;
    const bool in = k < p.d_ff && (p.force_all || ((p.ubits[k >> 5] >> (k & 31)) & 1u));
    int tot = 0;
    const int rank = block_exclusive_scan(in ? 1 : 0, &tot, sh);
    if (in) {
        p.lst[before + rank] = k;
        for (int w = 0; w < p.mw; ++w) {
            uint32_t m = 0;
            const int t1 = min(p.n, 32 * w + 32);
            for (int t = 32 * w; t < t1; ++t) {
                const long long zi = (long long)t * p.d_ff + k;
                const bool s = p.topk ? p.sel[zi] != 0 : p.z[zi] > p.tau;
                m |= (s ? 1u : 0u) << (t - 32 * w);
            }
            p.lst_mask[(size_t)k * p.mw + w] = m;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.u_count = total;
}

SmemAttrCache g_tc_smem;

}  // namespace

size_t tc_smem_bytes(int a_sub, int ks, int nb, int* stages) {
    const size_t stage = (size_t)a_sub * kTileA + (size_t)ks * nb * 128;
    int s = (int)((kMaxSmemPerCta - 1024 - sizeof(TcShared)) / stage);
    if (s > kMaxStages) s = kMaxStages;
    if (stages) *stages = s;
    if (s < 3) return 0;
    return 1024 + (size_t)s * stage + sizeof(TcShared);
}

cudaError_t launch_tc(const TcParams& p_in, int grid, cudaStream_t s, bool pdl) {
    TcParams p = p_in;
    if (p.nb < 16 || p.nb > 256 || p.nb % 16 || (p.paired && 2 * p.npad != p.nb)) return cudaErrorInvalidValue;
    // One 64-wide k-block and one 128-row accumulator tile per iteration: the
    // deepest ring of the smallest stages keeps the most bytes in flight.
    p.ks = 1;
    p.mt = 1;
    int st = 0;
    size_t smem = 0;
    for (;;) {
        smem = tc_smem_bytes(p.mode == kTcDown ? p.mt : p.ks, p.ks, p.nb, &st);
        if (smem || (p.ks == 1 && p.mt == 1)) break;
        if (p.ks > 1) p.ks >>= 1; else p.mt >>= 1;
    }
    if (!smem) return cudaErrorInvalidValue;
    p.stages = st;
    p.tmem_cols = 32;
    const int acc_cols = (p.mode == kTcDown ? p.mt : 1) * p.nb;
    while ((int)p.tmem_cols < 2 * acc_cols) p.tmem_cols <<= 1;
    if (p.tmem_cols > 512) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem(k_tc_gemm, smem, g_tc_smem);
    if (e != cudaSuccess) return e;
    return launch_ex(k_tc_gemm, dim3(grid), dim3(kTcThreads), smem, s, pdl, p);
}

cudaError_t launch_union(const UnionParams& p, cudaStream_t s, bool pdl) {
    const int grid = (p.d_ff + kUnionThreads - 1) / kUnionThreads;
    return launch_ex(k_union, dim3(grid), dim3(kUnionThreads), 0, s, pdl, p);
}

}  // namespace sffn
