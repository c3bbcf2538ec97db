// Batched path on the 5th-generation tensor cores (tcgen05).
//
// With several tokens per step the gate and the up and down passes are dense
// contractions of a token batch against weight rows, so they run as one
// tcgen05 GEMM kernel with four epilogues:
//
//   gate        Z^T[rows x n] = W[rows x K] . X^T        (z, fp32)
//   gate-split  the same, written as bf16 hi/lo rows      (LoPA: u = x A)
//   up          H^T[ch x n]   = W_up[ch] . X^T times the gate activation of ch
//   down        Y^T[d x n]    = W_down[ch]^T . H^T
//
// "Model Casting and Low-Parameter Gating" (abstract): gate first, then the
// other two matrices only where the activation is non-zero.
// "Mixture-of-Channels" (section "Dentro MoC"): rows of the channels the batch
// selected are loaded once and shared by the tokens that selected them; a
// token that did not select a channel gets a zero activation for it.
//
// The up and down passes read either whole 128-channel blocks or exactly the
// union's rows.  Blocks: every block holding a channel that some token of the
// batch selected (each CTA finds them from the gate's union bitmap; a channel
// of such a block that no token selected gets g = 0), in tiles the TMA engine
// moves with one instruction.  With several independent tokens nearly every
// block holds one.  Gathered rows: a one-CTA kernel lists the union's channels
// in ascending order, the A tiles are assembled four rows per TMA copy
// (tile::gather4 with a one-row box, landing in the same 128-byte-swizzled
// layout), h is kept in list order, and the down pass reduces over list
// positions.  A gathered row moves at about half the rate of a block tile, so
// a launch gathers only when the union holds under half of the channels
// (batches of a few tokens at high sparsity), decided on the device from the
// union's size.
//
// Kernel structure (one CTA per SM, 416 threads):
//   warps 0, 6 .. 12  one thread each: the TMA producers, P of them (4 for
//              tile passes, 8 for gathered ones).  Producer p fills the ring
//              stages of the k-blocks g with g % P == p: 2-D tile copies
//              (cp.async.bulk.tensor, 128-byte swizzle, no multicast) of the
//              A and B tiles, or four-row gathers of A, on mbarriers;
//   warp 1     allocates tensor memory; one thread issues tcgen05.mma (M = 128,
//              N = token columns, K = 16 per instruction, bf16 in, fp32
//              accumulate in tensor memory) and tcgen05.commit;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp its 32 TMEM
//              lanes), the mode's epilogue, stores.
// Work is split stream-K: the (tile, k-block) iterations are cut into one
// contiguous range per CTA, so every SM streams the same number of weight
// bytes.  A tile cut between CTAs is finished by the CTA holding its first
// k-blocks (at the end of that CTA's range), which adds the other CTAs' parts,
// parked early in their ranges, in CTA order: results are deterministic and
// the end of a range waits only for parts written long before.
//
// fp32 intermediates that feed a later MMA (LoPA's u = x A, and h) are passed
// as two bf16 rows, hi = bf16(v) and lo = bf16(v - hi); the MMA multiplies both
// and the epilogue adds the two columns, which keeps about 16 significant bits.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace sffn {
namespace {

constexpr int kBM = 128;            // accumulator rows (MMA M)
constexpr int kBK = 64;             // k-block: 64 bf16 = one 128-byte swizzle row
constexpr int kProdWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;        // epilogue warps 2..5
constexpr int kEpi = 4;
constexpr int kProdWarp2 = kEpiWarp0 + kEpi;   // further TMA producers: warps 6, 7, ...
constexpr int kMaxProducers = 8;   // gathered passes: up to 8; tile passes: 4
constexpr int kTcThreads = (kProdWarp2 + kMaxProducers - 1) * 32;
constexpr uint32_t kTileA = kBM * kBK * 2;   // 16 KB
constexpr int kMaxStages = 12;
constexpr int kMaxBlocks = 1024;    // 128-channel blocks (d_ff <= 131072)
constexpr int kMinIters = 8;        // iterations per CTA at least
constexpr int kMaxParts = 8;        // CTAs sharing one tile at most
constexpr int kIdxPerProducer = 2;  // gather: channel-index blocks each producer keeps in flight
constexpr int kIdxSlots = kMaxProducers * kIdxPerProducer;

struct TcShared {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t fix;           // the owner's staged copy of the other parts of its cut tile
    uint32_t tmem_base;
    int abort;
    int reducer;
    int wcount[kTcThreads / 32];
    int ucount;             // gather: the union's size
    int gmode;              // this launch gathers rows (the union is under half the channels)
    int nprod;              // producer threads taking turns over the k-blocks (<= the stages)
    int blk[kMaxBlocks];    // up/down: the active 128-channel blocks
    uint64_t ibar[kIdxSlots];
    alignas(16) int idx[kIdxSlots][kBM];   // gather: channel indices of one k-block's rows
};

// ---- tcgen05 / TMA primitives ------------------------------------------------

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
// 2-D tile of the tensor map at element coordinates (x = column, y = row) into
// this CTA's shared memory (1024-byte aligned), completing on `bar`.
// x is a multiple of 64 elements (128 bytes).
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
// Four rows of a one-row-box tensor map (rows r0..r3, columns x .. x + box)
// into four consecutive 128-byte rows of this CTA's shared memory at dst (the
// 128-byte swizzle follows the destination address, as for a tile), completing
// on `bar`.  x is a multiple of 64 elements (128 bytes).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, int x, int4 r, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(r.x), "r"(r.y), "r"(r.z), "r"(r.w),
          "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
// Ask the TMA engine to bring the box at (x, y) of the tensor map into L2.
__device__ __forceinline__ void tma_prefetch_tile(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
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


// The CTA c whose range [floor(c I/C), floor((c+1) I/C)) holds iteration i
// (C <= I, so no range is empty).
__device__ __forceinline__ int cta_of(long long i, long long I, int C) {
    return (int)(((i + 1) * C - 1) / I);
}

struct Seg {
    int t, kb0, kb1;
};

struct Problem {
    int T, KB, nblk;
    int C;                  // CTAs that take work
    long long I, it0, it1;
};

// nblk: the active 128-channel blocks, or when gathering the union's size.
__device__ __forceinline__ Problem make_problem(const TcParams& p, int nblk, bool gmode = false) {
    Problem q;
    q.nblk = nblk;
    if (p.mode == kTcUp) {
        q.T = gmode ? (nblk + kBM - 1) / kBM : q.nblk;
        q.KB = (p.k_total + kBK - 1) / kBK;
    } else if (p.mode == kTcDown) {
        q.T = (p.m_total + kBM - 1) / kBM;
        q.KB = gmode ? (nblk + kBK - 1) / kBK : 2 * q.nblk;
    } else {
        q.T = (p.m_total + kBM - 1) / kBM;
        q.KB = (p.k_total + kBK - 1) / kBK;
    }
    q.I = (long long)q.T * q.KB;
    q.C = (int)min(min((long long)gridDim.x, (q.I + kMinIters - 1) / kMinIters), (long long)q.T * kMaxParts);
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

// Before the wait for the previous kernel: the weight boxes of this CTA's first
// `count` k-blocks into L2, so the ring fills from L2 once the wait ends.
// Weights do not depend on earlier kernels.  The up and down passes do not know
// their active blocks yet; they take the boxes of the case where every block
// is active, which is the usual one with several tokens (a wrong guess costs
// only the prefetched bytes).
__device__ void prefetch_first_tiles(const TcParams& p, int count) {
    const bool blocks = p.mode == kTcUp || p.mode == kTcDown;
    const Problem q = make_problem(p, blocks ? (p.d_ff + 127) / 128 : 0);
    long long it = q.it0;
    int done = 0;
    Seg s;
    while (done < count && next_seg(q, it, s)) {
        for (int kb = s.kb0; kb < s.kb1 && done < count; ++kb, ++done) {
            if (p.mode == kTcDown) {
                const int c0 = (kb >> 1) * kBM + (kb & 1) * kBK;
                tma_prefetch_tile(&p.ta, s.t * kBM, c0);
                tma_prefetch_tile(&p.ta, s.t * kBM + 64, c0);
            } else {
                tma_prefetch_tile(&p.ta, kb * kBK, s.t * kBM);
            }
        }
    }
}

// ---- producer: one thread issues the TMA copies --------------------------------

// Producer `pr` of P = sh->nprod fills the stages of the k-blocks g with
// g % P == pr.  One thread issuing every copy of an SM's stream keeps only
// about three quarters of HBM bandwidth busy; threads in different warps,
// taking turns over the k-blocks of the same ring, reach the copy peak with
// tile copies.  A gathered stage takes 32 four-row copies, and the copy rate
// grows with the issuing threads: about 3 TB/s with four, 4 TB/s with eight.
// The ring stays one sequence for the MMA issuer.  (A producer waits for stage
// g - S to be consumed; with P <= S the parity wait cannot be a phase behind.)
// Gather: k-block g of the CTA's range is iteration it0 + g, i.e. tile
// (it0 + g) / KB and k-block (it0 + g) % KB, so a producer knows every future
// k-block's rows.  Their channel indices (up: the tile's 128 list entries;
// down: the k-block's 64) are bulk-copied into a small ring of index blocks,
// kIdxPerProducer k-blocks ahead of their use.
__device__ __forceinline__ void gather_index_copy(const TcParams& p, const Problem& q, TcShared* sh, int pr,
                                                  long long g) {
    const long long j = g / sh->nprod;
    const int slot = pr * kIdxPerProducer + (int)(j % kIdxPerProducer);
    const long long it = q.it0 + g;
    const int t = (int)(it / q.KB), kb = (int)(it % q.KB);
    const int* src = p.mode == kTcUp ? p.ulist + (size_t)t * kBM : p.ulist + (size_t)kb * kBK;
    const uint32_t bytes = p.mode == kTcUp ? kBM * 4u : kBK * 4u;
    mbar_expect_tx(&sh->ibar[slot], bytes);
    bulk_load(sh->idx[slot], src, bytes, &sh->ibar[slot], l2_evict_last());
}

__device__ void run_producer_gather(const TcParams& p, const Problem& q, unsigned char* stages, uint32_t stage_bytes,
                                    TcShared* sh, int pr) {
    const uint64_t pol_w = l2_evict_first(), pol_b = l2_evict_last();
    const int S = p.stages;
    const int NP = sh->nprod;
    if (pr >= NP) return;
    const uint32_t tx = kTileA + (uint32_t)p.nb * 128u;
    const long long n_it = q.it1 - q.it0;
    for (int j = 0; j < kIdxPerProducer; ++j) {
        const long long g = pr + (long long)NP * j;
        if (g < n_it) gather_index_copy(p, q, sh, pr, g);
    }
    for (long long g = pr; g < n_it; g += NP) {
        const long long j = g / NP;
        const int slot = pr * kIdxPerProducer + (int)(j % kIdxPerProducer);
        const long long it = q.it0 + g;
        const int t = (int)(it / q.KB), kb = (int)(it % q.KB);
        const int st = (int)(g % S);
        if (!mbar_wait_one(&sh->ibar[slot], (uint32_t)((j / kIdxPerProducer) & 1)) ||
            !mbar_wait_one(&sh->empty[st], (uint32_t)(((g / S) & 1) ^ 1))) {
            sh->abort = 1;
            raise_status(p.status, p.hstatus, kStatusWaitTimeout);
            return;
        }
        const uint32_t sA = smem_addr(stages + (size_t)st * stage_bytes);
        const uint32_t sB = sA + kTileA;
        const int4* rows = reinterpret_cast<const int4*>(sh->idx[slot]);
        if (p.mode == kTcDown) {
            // MN-major A: the k-block's 64 channels (rows of W_down) x 128 output columns, two 64-column
            // halves; a half wholly past the last output column is not loaded (its accumulator rows are
            // never stored, and each row of the product depends on its own A row only)
            const int m0 = t * kBM;
            const bool hi = m0 + 64 < p.m_total;
            mbar_expect_tx(&sh->full[st], hi ? tx : tx - 8192u);
#pragma unroll 4
            for (int i = 0; i < kBK / 4; ++i) {
                const int4 r = rows[i];
                tma_gather4(sA + i * 512, &p.tg, m0, r, &sh->full[st], pol_w);
                if (hi) tma_gather4(sA + 8192 + i * 512, &p.tg, m0 + 64, r, &sh->full[st], pol_w);
            }
            tma_tile(sB, &p.tb, kb * kBK, 0, &sh->full[st], pol_b);   // h, compacted by list position
        } else {
            // K-major A: the tile's 128 channels (rows of W_up) x 64 k
            mbar_expect_tx(&sh->full[st], tx);
#pragma unroll 4
            for (int i = 0; i < kBM / 4; ++i) tma_gather4(sA + i * 512, &p.tg, kb * kBK, rows[i], &sh->full[st], pol_w);
            tma_tile(sB, &p.tb, kb * kBK, 0, &sh->full[st], pol_b);
        }
        // this thread's reads of the index block come before the async copy that refills it
        fence_proxy_async();
        const long long gn = g + (long long)NP * kIdxPerProducer;
        if (gn < n_it) gather_index_copy(p, q, sh, pr, gn);
    }
}

__device__ void run_producer(const TcParams& p, const Problem& q, unsigned char* stages, uint32_t stage_bytes,
                             TcShared* sh, int pr) {
    if (sh->gmode) {
        run_producer_gather(p, q, stages, stage_bytes, sh, pr);
        return;
    }
    const uint64_t pol_w = l2_evict_first(), pol_b = l2_evict_last();
    const int S = p.stages;
    const int NP = sh->nprod;
    if (pr >= NP) return;
    const uint32_t tx = kTileA + (uint32_t)p.nb * 128u;
    long long it = q.it0, g = 0;
    Seg s;
    while (next_seg(q, it, s)) {
        const int m0 = p.mode == kTcUp ? sh->blk[s.t] * kBM : s.t * kBM;
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++g) {
            if ((int)(g % NP) != pr) continue;
            const int st = (int)(g % S);
            if (!mbar_wait_one(&sh->empty[st], (uint32_t)(((g / S) & 1) ^ 1))) {
                sh->abort = 1;
                raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                return;
            }
            const uint32_t sA = smem_addr(stages + (size_t)st * stage_bytes);
            const uint32_t sB = sA + kTileA;
            mbar_expect_tx(&sh->full[st], tx);
            if (p.mode == kTcDown) {
                // MN-major A: 64 channels (k) x 128 output columns (m) of W_down, two 64-column boxes
                const int c0 = sh->blk[kb >> 1] * kBM + (kb & 1) * kBK;
                tma_tile(sA, &p.ta, m0, c0, &sh->full[st], pol_w);
                tma_tile(sA + 8192, &p.ta, m0 + 64, c0, &sh->full[st], pol_w);
                tma_tile(sB, &p.tb, c0, 0, &sh->full[st], pol_b);
            } else {
                tma_tile(sA, &p.ta, kb * kBK, m0, &sh->full[st], pol_w);
                tma_tile(sB, &p.tb, kb * kBK, 0, &sh->full[st], pol_b);
            }
        }
    }
}

// ---- MMA issuer --------------------------------------------------------------

__device__ void run_mma(const TcParams& p, const Problem& q, unsigned char* stages, uint32_t stage_bytes,
                        TcShared* sh, uint32_t tmem) {
    const int S = p.stages;
    const bool down = p.mode == kTcDown;
    const uint32_t idesc = mma_idesc(p.nb, down ? 1 : 0);
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
        const uint32_t d_tmem = tmem + (uint32_t)(acc * p.nb);
        for (int kb = s.kb0; kb < s.kb1; ++kb, ++g) {
            const int st = (int)(g % S);
            if (!mbar_wait_one(&sh->full[st], (uint32_t)((g / S) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sA = smem_addr(stages + (size_t)st * stage_bytes);
            const uint32_t sB = sA + kTileA;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint64_t ad =
                    down ? sw128_desc(sA + kk * 2048, 8192, 1024) : sw128_desc(sA + kk * 32, 16, 1024);
                tc_mma(d_tmem, ad, sw128_desc(sB + kk * 32, 16, 1024), idesc, (kb > s.kb0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&sh->empty[st]);
        }
        if (!ok) break;
        tc_commit(&sh->tfull[acc]);
        ++segi;
    }
    if (!ok) {
        sh->abort = 1;
        raise_status(p.status, p.hstatus, kStatusWaitTimeout);
    }
    // all issued MMAs complete before the accumulators are released
    tc_commit(&sh->drain);
    mbar_wait_one(&sh->drain, 0);
}

// ---- epilogue ----------------------------------------------------------------

// Final values v[0..15] of columns c0..c0+15 (hi+lo combined when paired) of
// output row m.  `act` collects the gate's activity flag.
__device__ __forceinline__ void emit16(const TcParams& p, int m, int c0, const float* v, bool& act) {
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

// ---- up epilogue ---------------------------------------------------------------
// h(token, m) = g(token, m) * acc, g the gate activation of channel m for the
// token (ReLU(z - tau), or the selected SiLU value; zero past n and d_ff).
// The gate values of a tile's first kUpChunks x 16 tokens are loaded into
// registers before its accumulator is ready, so their latency hides behind
// the mainloop; the values of later tokens (passes of up to 256) are loaded
// one chunk ahead of their use.

constexpr int kUpChunks = 4;

struct UpG {
    float raw[kUpChunks * 16];
};

// The 16 gate values of channel m (m < 0: none, a padding row of a gathered
// tile) for token columns 16j .. 16j + 15.
__device__ __forceinline__ void up_g_chunk(const TcParams& p, int m, int j, float* g16) {
    const float* src = p.topk ? p.gsel : p.zsel;
    const bool row_ok = m >= 0 && m < p.m_total;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int tok = 16 * j + i;
        g16[i] = (row_ok && tok < p.n) ? __ldcg(src + (long long)tok * p.ldsel + m) : 0.f;
    }
}

// Issue the loads of the gate values of channel m for the first `cols` token
// columns (at most kUpChunks x 16).
__device__ __forceinline__ void up_g_load(const TcParams& p, int m, int cols, UpG& g) {
#pragma unroll
    for (int j = 0; j < kUpChunks; ++j)
        if (16 * j < cols) up_g_chunk(p, m, j, g.raw + 16 * j);
}

// Columns 16j..16j+15 of channel m (m < 0: a padding row, h = 0): h = g * v,
// written as bf16 rows (and, for a paired consumer, the rounding remainder as
// lo rows) at output column mo (the channel, or with gather its list
// position).  g16: the 16 gate values of those columns.
__device__ __forceinline__ void up_emit16(const TcParams& p, int m, int mo, int j, const float* v,
                                          const float* g16) {
    bf16* o = static_cast<bf16*>(p.out);
    const bool row_ok = m >= 0 && m < p.m_total;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int tok = 16 * j + i;
        const float raw = g16[i];
        const float gv = (row_ok && tok < p.n) ? (p.topk ? raw : fmaxf(raw - p.tau, 0.f)) : 0.f;
        const float h = row_ok ? gv * v[i] : 0.f;
        const bf16 hi = __float2bfloat16_rn(h);
        o[(long long)tok * p.ldo + mo] = hi;
        if (p.h_pairs) o[(long long)(p.npad + tok) * p.ldo + mo] = __float2bfloat16_rn(h - __bfloat162float(hi));
    }
}

// ---- stream-K fix-up ----------------------------------------------------------
// A tile cut between CTAs c_first < ... < c_last: c_first holds the tile's first
// k-blocks, at the end of its range (its last segment), and owns the tile.  Every
// later CTA holds the tile in its first (or only) segment and parks its partial
// accumulator in its part slot early in its run.  The owner adds those parts, in
// CTA order, to its own accumulator and finishes the tile as it would a whole
// one.  So the only wait at the end of a range is for parts that are normally
// written long before, no CTA waits for a range that ends as late as its own,
// and the owner's partial sum never goes through memory.  The waits point to
// higher CTA indices only, so they cannot form a cycle.

// Parts are parked row-major (row = TMEM lane, nb floats: the hi columns, then
// the lo), with the 16-byte chunks of each row permuted by an XOR with the row
// index, so the 32 rows a warp reads at one column sit in different banks once
// staged in shared memory.
__device__ __forceinline__ int part_swz_mask(int nb) {
    const int q4 = nb >> 2;               // a multiple of 4
    return min(q4 & -q4, 8) - 1;
}

// v[0..15] += the np parts at base, base + stride, ... (in that order) at
// columns c0..c0+15 of row `row` (each part's hi + lo columns when paired).
// `global` selects L2 loads (parts still in global memory) over plain loads
// (parts staged in shared memory).
__device__ __forceinline__ void add_parts16(const TcParams& p, const float* base, size_t stride, int np, int row,
                                            int c0, bool global, float* v) {
    const int mask = part_swz_mask(p.nb);
    for (int k = 0; k < np; ++k) {
        const float4* r4 = reinterpret_cast<const float4*>(base + (size_t)k * stride + (size_t)row * p.nb);
        float4 a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int ja = ((c0 >> 2) + i) ^ (row & mask);
            const int jb = ((p.npad + c0) >> 2) + i;
            a[i] = global ? __ldcg(r4 + ja) : r4[ja];
            b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.paired) b[i] = global ? __ldcg(r4 + (jb ^ (row & mask))) : r4[jb ^ (row & mask)];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i] += a[i].x + b[i].x;
            v[4 * i + 1] += a[i].y + b[i].y;
            v[4 * i + 2] += a[i].z + b[i].z;
            v[4 * i + 3] += a[i].w + b[i].w;
        }
    }
}

// The owner's wait (bounded) until `want` parts of tile t have arrived.
__device__ __forceinline__ bool wait_parts(const TcParams& p, int t, unsigned want) {
    const unsigned* arrivals = p.tickets + 2 * t;
    bool ready = true;
    if ((threadIdx.x & 31) == 0 && ld_acquire(arrivals) < want) {
        const unsigned long long t0 = globaltimer_ns();
        unsigned backoff = 32;
        while (ld_acquire(arrivals) < want) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                ready = false;
                break;
            }
            __nanosleep(backoff);
            if (backoff < 256) backoff <<= 1;
        }
    }
    ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
    __threadfence();
    return ready;
}

__device__ void run_epilogue(const TcParams& p, const Problem& q, TcShared* sh, uint32_t tmem,
                             unsigned char* ring, size_t ring_bytes) {
    const int warp = threadIdx.x >> 5;
    const int quarter = warp & 3;                     // TMEM lanes this warp may access
    const int lane = threadIdx.x & 31;
    const int row = quarter * 32 + lane;
    const int etid = threadIdx.x - kEpiWarp0 * 32;    // 0..127
    const int cols = p.paired ? p.npad : p.nb;        // final columns
    const int C = q.C;
    const size_t slot_floats = (size_t)p.nb * kBM;
    long long it = q.it0;
    int segi = 0;
    Seg s;
    while (next_seg(q, it, s)) {
        const int acc = segi & 1;
        const uint32_t use = (uint32_t)(segi >> 1);
        ++segi;
        const bool whole = s.kb0 == 0 && s.kb1 == q.KB;
        const int c_first = whole ? (int)blockIdx.x : cta_of((long long)s.t * q.KB, q.I, C);
        const int c_last = whole ? (int)blockIdx.x : cta_of((long long)(s.t + 1) * q.KB - 1, q.I, C);
        const bool owner = c_first == (int)blockIdx.x;
        // up: output row `row` of the tile is channel m, written at column mo
        // (gather: list position mo = the tile's first position + row, whose
        // channel is the list entry, none past the union's size)
        const int m0 = p.mode == kTcUp ? (sh->gmode ? s.t * kBM : sh->blk[s.t] * kBM) : s.t * kBM;
        const int mo = m0 + row;
        const int m = (p.mode == kTcUp && sh->gmode) ? (mo < sh->ucount ? __ldcg(p.ulist + mo) : -1) : mo;
        UpG g;
        if (p.mode == kTcUp && owner) up_g_load(p, m, cols, g);   // in flight during the mainloop
        if (owner && !whole && !wait_parts(p, s.t, (unsigned)(c_last - c_first))) {
            sh->abort = 1;
            raise_status(p.status, p.hstatus, kStatusWaitTimeout);
            return;
        }
        if (!mbar_wait_warp(&sh->tfull[acc], use & 1u)) {
            sh->abort = 1;
            raise_status(p.status, p.hstatus, kStatusWaitTimeout);
            return;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.nb);
        if (owner) {
            // the other parts: staged into the (now idle) stage ring with bulk copies
            // when they fit, else read from L2 chunk by chunk
            const int np = c_last - c_first;
            const float* pbase = p.part + (size_t)(c_first + 1) * slot_floats;
            bool pglobal = true;
            if (np > 0 && (size_t)np * slot_floats * 4 <= ring_bytes) {
                // the last segment's accumulator is complete, so every MMA has read
                // its stages and no copy into the ring is in flight
                if (etid == 0) {
                    const uint32_t bytes = (uint32_t)((size_t)np * slot_floats * 4);
                    const uint64_t pol = l2_evict_first();
                    fence_proxy_async_global();
                    mbar_expect_tx(&sh->fix, bytes);
                    for (uint32_t o = 0; o < bytes; o += 16384u)
                        bulk_load(ring + o, reinterpret_cast<const unsigned char*>(pbase) + o,
                                  min(16384u, bytes - o), &sh->fix, pol);
                }
                if (!mbar_wait_warp(&sh->fix, 0)) {
                    sh->abort = 1;
                    raise_status(p.status, p.hstatus, kStatusWaitTimeout);
                    return;
                }
                pbase = reinterpret_cast<const float*>(ring);
                pglobal = false;
            }
            bool act = false;
            if (p.mode == kTcUp) {
#pragma unroll
                for (int j = 0; j < kUpChunks; ++j) {
                    if (16 * j >= cols) break;
                    float v[16];
                    tmem_ld16(taddr + 16 * j, v);
                    add_parts16(p, pbase, slot_floats, np, row, 16 * j, pglobal, v);
                    up_emit16(p, m, mo, j, v, g.raw + 16 * j);
                }
                if (cols > 16 * kUpChunks) {
                    // tokens past the preloaded ones: each chunk's gate values load
                    // while the previous chunk's accumulator is read and emitted
                    float gn[16];
                    up_g_chunk(p, m, kUpChunks, gn);
                    for (int j = kUpChunks; 16 * j < cols; ++j) {
                        float gc[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) gc[i] = gn[i];
                        if (16 * (j + 1) < cols) up_g_chunk(p, m, j + 1, gn);
                        float v[16];
                        tmem_ld16(taddr + 16 * j, v);
                        add_parts16(p, pbase, slot_floats, np, row, 16 * j, pglobal, v);
                        up_emit16(p, m, mo, j, v, gc);
                    }
                }
            } else {
                for (int c0 = 0; c0 < cols; c0 += 16) {
                    float v[16];
                    tmem_ld16(taddr + c0, v);
                    if (p.paired) {
                        float x[16];
                        tmem_ld16(taddr + p.npad + c0, x);
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] += x[i];
                    }
                    add_parts16(p, pbase, slot_floats, np, row, c0, pglobal, v);
                    emit16(p, m, c0, v, act);
                    if (p.mode == kTcGateZ && p.selbits && !p.topk) {
                        // the selection itself, per token: one word per 32 channels of this warp
                        const bool word_ok = m0 + quarter * 32 < p.m_total;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int tok = c0 + i;
                            const unsigned b = __ballot_sync(0xffffffffu, tok < p.n && m < p.m_total && v[i] > p.tau);
                            if (lane == 0 && word_ok && tok < p.n)
                                p.selbits[(long long)tok * p.selw + ((m0 + quarter * 32) >> 5)] = b;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sh->tempty[acc]);
            if (p.mode == kTcGateZ && p.ubits) {
                // union bitmap words of this tile: one word per warp (32 channels)
                const unsigned bits = __ballot_sync(0xffffffffu, act && !p.topk && m < p.m_total);
                if (lane == 0) p.ubits[(m0 + quarter * 32) >> 5] = bits;
            }
            if (!whole) {
                // the last of the owner's four warps resets the tile's counters for the next launch
                __syncwarp();
                unsigned* arrivals = p.tickets + 2 * s.t;
                if (lane == 0 && atomicAdd(arrivals + 1, 1u) == 3u) {
                    arrivals[0] = 0u;
                    arrivals[1] = 0u;
                }
            }
        } else {
            // a later part of a cut tile: park it for the owner
            float4* mine = reinterpret_cast<float4*>(p.part + (size_t)blockIdx.x * slot_floats + (size_t)row * p.nb);
            const int mask = part_swz_mask(p.nb);
            for (int c0 = 0; c0 < p.nb; c0 += 16) {
                float v[16];
                tmem_ld16(taddr + c0, v);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    mine[((c0 >> 2) + i) ^ (row & mask)] =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            tc_fence_before();
            mbar_arrive(&sh->tempty[acc]);
            fence_proxy_async_global();   // the owner may read the part with bulk copies
            __threadfence();
            named_sync(1, kEpi * 32);
            if (etid == 0) atomicAdd(p.tickets + 2 * s.t, 1u);
        }
    }
}

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_gemm(const __grid_constant__ TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* stages = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                             ~static_cast<uintptr_t>(1023));
    const uint32_t stage_bytes = kTileA + (uint32_t)p.nb * 128u;
    TcShared* sh = reinterpret_cast<TcShared*>(stages + (size_t)p.stages * stage_bytes);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) {
            mbar_init(&sh->full[i], 1);
            mbar_init(&sh->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->tfull[i], 1);
            mbar_init(&sh->tempty[i], kEpi * 32);
        }
        mbar_init(&sh->drain, 1);
        mbar_init(&sh->fix, 1);
        for (int i = 0; i < kIdxSlots; ++i) mbar_init(&sh->ibar[i], 1);
        sh->abort = 0;
        sh->reducer = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&sh->tmem_base, p.tmem_cols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == kProdWarp && (threadIdx.x & 31) == 0) prefetch_first_tiles(p, p.stages);
    griddep_launch_dependents();
    griddep_wait();
    int nblk = 0;
    // Gathering the union's rows moves fewer bytes but at about half the rate
    // of whole-block tiles (four rows per copy instead of 128), so it is taken
    // only when the union holds under half of the channels.
    const int U = p.gather ? __ldcg(p.ucount) : 0;
    const bool gmode = p.gather && 2 * U < p.d_ff;
    if (threadIdx.x == 0) {
        sh->ucount = U;
        sh->gmode = gmode ? 1 : 0;
        sh->nprod = min(gmode ? kMaxProducers : 4, p.stages);
    }
    __syncthreads();
    if (gmode) {
        nblk = U;                                      // its list was built by the previous kernel
    } else if (p.mode == kTcUp || p.mode == kTcDown) {
        // the 128-channel blocks holding a channel some token selected, from the union bitmap
        const int nbk = (p.d_ff + 127) / 128, nwords = (p.d_ff + 31) >> 5;
        const int lane = threadIdx.x & 31;
        for (int b0 = 0; b0 < nbk; b0 += kTcThreads) {
            const int bi = b0 + threadIdx.x;
            bool act = false;
            if (bi < nbk) {
                if (p.force_all) {
                    act = true;
                } else {
                    for (int w = 4 * bi; w < min(4 * bi + 4, nwords); ++w) {
                        uint32_t bits = __ldcg(p.ubits + w);
                        if (w == nwords - 1 && (p.d_ff & 31)) bits &= (1u << (p.d_ff & 31)) - 1u;
                        act |= bits != 0u;
                    }
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, act);
            if (lane == 0) sh->wcount[warp] = __popc(m);
            __syncthreads();
            int before = nblk;
            for (int w2 = 0; w2 < warp; ++w2) before += sh->wcount[w2];
            if (act) sh->blk[before + __popc(m & ((1u << lane) - 1u))] = bi;
            for (int w2 = 0; w2 < kTcThreads / 32; ++w2) nblk += sh->wcount[w2];
            __syncthreads();
        }
    }
    const Problem q = make_problem(p, nblk, gmode);
    if (p.mode == kTcDown && q.KB == 0) {
        // no channel is active for any token: y = 0
        bf16* y = static_cast<bf16*>(p.out);
        const long long total = (long long)p.n * p.m_total;
        for (long long i = (long long)blockIdx.x * kTcThreads + threadIdx.x; i < total;
             i += (long long)gridDim.x * kTcThreads) {
            const long long t = i / p.m_total;
            y[t * p.ldo + (i - t * p.m_total)] = __float2bfloat16_rn(0.f);
        }
    }

    if (warp == kProdWarp || warp >= kProdWarp2) {
        if ((threadIdx.x & 31) == 0)
            run_producer(p, q, stages, stage_bytes, sh, warp == kProdWarp ? 0 : warp - kProdWarp2 + 1);
    } else if (warp == kMmaWarp) {
        if ((threadIdx.x & 31) == 0) run_mma(p, q, stages, stage_bytes, sh, tmem);
    } else {
        run_epilogue(p, q, sh, tmem, stages, (size_t)p.stages * stage_bytes);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, p.tmem_cols);
}

// The union bitmap as an ascending channel list (one CTA): each thread takes a
// run of words, a block scan places them, and the list is padded with channel
// 0 (a real row, whose h is zero) to a multiple of 128 for the gathered tiles.
constexpr int kListThreads = 1024;
__global__ void __launch_bounds__(kListThreads) k_union_list(const uint32_t* ubits, int d_ff, int* list, int* count) {
    __shared__ int sh[40];
    griddep_wait();
    griddep_launch_dependents();
    const int W = (d_ff + 31) >> 5;
    const int per = (W + kListThreads - 1) / kListThreads;
    const int w0 = min(W, (int)threadIdx.x * per), w1 = min(W, w0 + per);
    auto word = [&](int w) {
        uint32_t b = __ldcg(ubits + w);
        if (w == W - 1 && (d_ff & 31)) b &= (1u << (d_ff & 31)) - 1u;
        return b;
    };
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(word(w));
    int U = 0;
    int pos = block_exclusive_scan(c, &U, sh);
    for (int w = w0; w < w1; ++w) {
        uint32_t b = word(w);
        while (b) {
            list[pos++] = 32 * w + __ffs(b) - 1;
            b &= b - 1u;
        }
    }
    const int padded = (U + kBM - 1) / kBM * kBM;
    for (int i = U + (int)threadIdx.x; i < padded; i += kListThreads) list[i] = 0;
    if (threadIdx.x == 0) *count = U;
}

SmemAttrCache g_tc_smem;
std::once_flag g_enc_once;
PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;

}  // namespace

size_t tc_smem_bytes(int nb, int* stages) {
    const size_t stage = kTileA + (size_t)nb * 128;
    int s = (int)((kMaxSmemPerCta - 1024 - sizeof(TcShared)) / stage);
    if (s > kMaxStages) s = kMaxStages;
    if (stages) *stages = s;
    if (s < 3) return 0;
    return 1024 + (size_t)s * stage + sizeof(TcShared);
}

cudaError_t launch_union_list(const uint32_t* ubits, int d_ff, int* list, int* count, cudaStream_t s, bool pdl) {
    if (!ubits || !list || !count || d_ff < 1) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kListThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_union_list, ubits, d_ff, list, count);
}

cudaError_t launch_tc(const TcParams& p_in, int grid, cudaStream_t s, bool pdl) {
    TcParams p = p_in;
    if (p.nb < 16 || p.nb > 256 || p.nb % 16 || (p.paired && 2 * p.npad != p.nb)) return cudaErrorInvalidValue;
    if ((p.mode == kTcUp || p.mode == kTcDown) && ((p.d_ff + 127) / 128 > kMaxBlocks || (!p.ubits && !p.force_all)))
        return cudaErrorInvalidValue;
    if (p.gather && (!p.ulist || !p.ucount || (p.mode != kTcUp && p.mode != kTcDown))) return cudaErrorInvalidValue;
    int st = 0;
    const size_t smem = tc_smem_bytes(p.nb, &st);
    if (!smem) return cudaErrorInvalidValue;
    p.stages = st;
    p.tmem_cols = 32;
    while ((int)p.tmem_cols < 2 * p.nb) p.tmem_cols <<= 1;
    cudaError_t e = ensure_smem(k_tc_gemm, smem, g_tc_smem);
    if (e != cudaSuccess) return e;
    return launch_ex(k_tc_gemm, dim3(grid), dim3(kTcThreads), smem, s, pdl, p);
}


// 2-D bf16 tensor map (row-major, `cols` contiguous elements per row) with a
// box of box_cols x box_rows elements and the 128-byte swizzle; elements
// outside the tensor read as zero.  The driver's encoder is fetched once
// through the runtime.
cudaError_t encode_tile_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                            uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows) {
    std::call_once(g_enc_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_enc) return cudaErrorNotSupported;
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_bytes & 15) || cols == 0 || rows == 0 ||
        box_cols * 2 > 128 || box_rows > 256)
        return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace sffn
