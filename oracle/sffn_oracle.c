/*
 * CPU oracle for the activation-sparse gated FFN.  TEST INFRASTRUCTURE ONLY:
 * the tests, the package's smoke check and the bench's CPU-baseline leg call
 * it; the library never does.  It shares no code with the CUDA path.
 *
 * What it computes (plain definitions, fp64, explicit loops, fixed order):
 *
 *   gated FFN          y = W_down^T ( act(x W_gate) (*) (x W_up) )
 *     "Model Casting and Low-Parameter Gating" (abstract): the gating matrix is
 *     evaluated first; where its activation is zero the two other matrices are
 *     not needed.  "Mixture-of-Channels" (section "Perche Mixture-of-Channels")
 *     names the gate/up pair as SwiGLU's.
 *   LoPA gate          W_gate = A B (rank r), evaluated as z = (x A) B
 *     "Model Casting and Low-Parameter Gating" (abstract: a low-FLOPs
 *     parameterization of the gating matrix).  Read here as a rank-r product.
 *   threshold select   S_t = { k : z[t,k] > tau },  g = z - tau on S_t
 *     (a shifted ReLU, the "sparsity inducing activation" of model casting)
 *   top-K select       S_t = the K channels with the largest SiLU(z[t,k]),
 *                      ties to the lower index;  g = SiLU(z) on S_t
 *   top-p select       S_t = the shortest prefix, by descending z (ties to the
 *                      lower index), whose softmax mass reaches p;  g = SiLU(z)
 *     "PrunePath" (abstract: softmax-normalised routing distribution,
 *     cumulative-mass threshold, token-level probability budget).
 *     "Mixture-of-Channels" (sections "Dentro il mixture", "Dentro MoC": Top-K
 *     channels per token, ranked by the SwiGLU gate).
 *   sparse FFN         y[t,:] = sum over k in S_t, ascending, of
 *                      g[t,k] * <x[t,:], W_up[:,k]> * W_down[k,:]
 *   dense FFN          the same sum over all d_ff channels with g = 0 off S_t
 *
 * Inputs are read in their storage type (bf16 bits, fp32 or fp64) and widened
 * exactly to double.  Layouts are the API's row-major ones: x n x d,
 * W_gate and W_up d x d_ff, W_down d_ff x d, A d x r, B r x d_ff.
 *
 * Every sum runs in ascending index order and threads only split independent
 * outputs, so results do not depend on the thread count.  Build with
 * -ffp-contract=off so that no fused multiply-add changes the rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ODT_BF16 = 0, ODT_F32 = 1, ODT_F64 = 2 };
enum { OSEL_THRESHOLD = 0, OSEL_TOPK = 1, OSEL_TOPP = 2 };

/* Exact widening of one stored element to double.  A bf16 value is the upper
 * half of an IEEE binary32, so its bits shifted left by 16 are that binary32. */
static inline double ld(const void* p, int dt, int64_t i) {
    if (dt == ODT_BF16) {
        uint32_t b = (uint32_t)((const uint16_t*)p)[i] << 16;
        float f;
        memcpy(&f, &b, sizeof f);
        return (double)f;
    }
    if (dt == ODT_F32) return (double)((const float*)p)[i];
    return ((const double*)p)[i];
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* out[t,c] = sum_{j ascending} in[t,j] * M[j,c]   (in: n x rows, M: rows x cols)
 * The vector-matrix product behind the dense gate, LoPA's two stages and the
 * dense up projection. */
void oracle_vecmat(const void* in, int in_dt, const void* M, int m_dt,
                   int64_t n, int64_t rows, int64_t cols, double* out) {
    const int64_t CB = 256;
    const int64_t nblk = (cols + CB - 1) / CB;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblk; b++) {
        const int64_t c0 = b * CB, c1 = c0 + CB < cols ? c0 + CB : cols;
        for (int64_t t = 0; t < n; t++) {
            double* o = out + t * cols;
            for (int64_t c = c0; c < c1; c++) o[c] = 0.0;
            for (int64_t j = 0; j < rows; j++) {
                const double v = ld(in, in_dt, t * rows + j);
                for (int64_t c = c0; c < c1; c++) o[c] += v * ld(M, m_dt, j * cols + c);
            }
        }
    }
}

/* Dense gate: z = x W_gate  (n x d_ff). */
void oracle_gate_dense(const void* x, int x_dt, const void* w_gate, int w_dt,
                       int64_t n, int64_t d, int64_t d_ff, double* z) {
    oracle_vecmat(x, x_dt, w_gate, w_dt, n, d, d_ff, z);
}

/* LoPA gate: u = x A (n x r, kept in fp64), then z = u B (n x d_ff). */
void oracle_gate_lopa(const void* x, int x_dt, const void* A, const void* B, int w_dt,
                      int64_t n, int64_t d, int64_t r, int64_t d_ff, double* u, double* z) {
    oracle_vecmat(x, x_dt, A, w_dt, n, d, r, u);
    oracle_vecmat(u, ODT_F64, B, w_dt, n, r, d_ff, z);
}

static inline double silu(double z) { return z / (1.0 + exp(-z)); }

/* The activation on a selected channel: z - tau (threshold) or SiLU(z) (top-K). */
static inline double act(double z, int kind, double tau) {
    return kind == OSEL_THRESHOLD ? z - tau : silu(z);
}

/* g[t,k] = act(z[t,k]) for every k listed for token t, 0 elsewhere.
 * idx holds token t's list at idx[t*d_ff .. t*d_ff + cnt[t]). */
void oracle_gate_values(const double* z, int64_t n, int64_t d_ff, const int32_t* idx,
                        const int32_t* cnt, int kind, double tau, double* g) {
    for (int64_t t = 0; t < n; t++) {
        double* gt = g + t * d_ff;
        for (int64_t k = 0; k < d_ff; k++) gt[k] = 0.0;
        for (int32_t p = 0; p < cnt[t]; p++) {
            const int32_t k = idx[t * d_ff + p];
            gt[k] = act(z[t * d_ff + k], kind, tau);
        }
    }
}

/* Threshold selection: S_t = { k : z[t,k] > tau } in ascending order. */
void oracle_select_threshold(const double* z, int64_t n, int64_t d_ff, double tau,
                             int32_t* idx, int32_t* cnt, double* g) {
    for (int64_t t = 0; t < n; t++) {
        int32_t c = 0;
        for (int64_t k = 0; k < d_ff; k++)
            if (z[t * d_ff + k] > tau) idx[t * d_ff + c++] = (int32_t)k;
        cnt[t] = c;
    }
    oracle_gate_values(z, n, d_ff, idx, cnt, OSEL_THRESHOLD, tau, g);
}

typedef struct { double key; int32_t k; } rank_item;

/* Descending key, then ascending channel index. */
static int by_key_desc(const void* a, const void* b) {
    const rank_item* x = (const rank_item*)a;
    const rank_item* y = (const rank_item*)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->k > y->k) - (x->k < y->k);
}

static int by_int_asc(const void* a, const void* b) {
    const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Top-K selection: rank channels by SiLU(z) (ties: lower index first), keep
 * the first K, and list them in ascending index order.  Returns -1 on a bad K
 * or an allocation failure. */
int oracle_select_topk(const double* z, int64_t n, int64_t d_ff, int64_t K,
                       int32_t* idx, int32_t* cnt, double* g) {
    if (K < 0 || K > d_ff) return -1;
    rank_item* items = (rank_item*)malloc(sizeof(rank_item) * (size_t)(d_ff > 0 ? d_ff : 1));
    if (!items) return -1;
    for (int64_t t = 0; t < n; t++) {
        for (int64_t k = 0; k < d_ff; k++) {
            items[k].key = silu(z[t * d_ff + k]);
            items[k].k = (int32_t)k;
        }
        qsort(items, (size_t)d_ff, sizeof(rank_item), by_key_desc);
        for (int64_t p = 0; p < K; p++) idx[t * d_ff + p] = items[p].k;
        qsort(idx + t * d_ff, (size_t)K, sizeof(int32_t), by_int_asc);
        cnt[t] = (int32_t)K;
    }
    free(items);
    oracle_gate_values(z, n, d_ff, idx, cnt, OSEL_TOPK, 0.0, g);
    return 0;
}

/* Top-p selection ("PrunePath", abstract: a softmax-normalised routing
 * distribution and a cumulative-mass threshold, i.e. a per-token probability
 * budget).  Per token: P_k = exp(z_k - max z) / sum_j exp(z_j - max z); rank
 * the channels by z (the order of P), ties to the lower index; keep the
 * shortest prefix whose mass reaches p; list it ascending.  p = 0 keeps none.
 * Activation SiLU(z) on the kept channels, as for top-K.  Returns -1 on p
 * outside [0, 1] or an allocation failure. */
int oracle_select_topp(const double* z, int64_t n, int64_t d_ff, double p,
                       int32_t* idx, int32_t* cnt, double* g) {
    if (!(p >= 0.0 && p <= 1.0)) return -1;
    rank_item* items = (rank_item*)malloc(sizeof(rank_item) * (size_t)(d_ff > 0 ? d_ff : 1));
    if (!items) return -1;
    for (int64_t t = 0; t < n; t++) {
        const double* zt = z + t * d_ff;
        int32_t c = 0;
        if (d_ff > 0 && p > 0.0) {
            double m = zt[0];
            for (int64_t k = 1; k < d_ff; k++) if (zt[k] > m) m = zt[k];
            double total = 0.0;
            for (int64_t k = 0; k < d_ff; k++) total += exp(zt[k] - m);
            for (int64_t k = 0; k < d_ff; k++) {
                items[k].key = zt[k];
                items[k].k = (int32_t)k;
            }
            qsort(items, (size_t)d_ff, sizeof(rank_item), by_key_desc);
            const double target = p * total;
            double cum = 0.0;
            for (int64_t q = 0; q < d_ff; q++) {
                idx[t * d_ff + c++] = items[q].k;
                cum += exp(items[q].key - m);
                if (cum >= target) break;
            }
            qsort(idx + t * d_ff, (size_t)c, sizeof(int32_t), by_int_asc);
        }
        cnt[t] = c;
    }
    free(items);
    oracle_gate_values(z, n, d_ff, idx, cnt, OSEL_TOPP, 0.0, g);
    return 0;
}

/* Sparse FFN on the listed channels only:
 *   u[t,k] = sum_j x[t,j] W_up[j,k]   for k in S_t
 *   y[t,:] = sum_{k in S_t ascending} (g[t,k] u[t,k]) W_down[k,:]
 * u_out (n x d_ff, may be NULL) receives u on S_t and 0 elsewhere. */
void oracle_sparse_ffn(const void* x, int x_dt, const void* w_up, const void* w_down, int w_dt,
                       int64_t n, int64_t d, int64_t d_ff, const int32_t* idx,
                       const int32_t* cnt, const double* g, double* y, double* u_out) {
    double* h = (double*)malloc(sizeof(double) * (size_t)(d_ff > 0 ? d_ff : 1));
    for (int64_t t = 0; t < n; t++) {
        const int32_t m = cnt[t];
        const int32_t* S = idx + t * d_ff;
#pragma omp parallel for schedule(static)
        for (int32_t p = 0; p < m; p++) {
            const int32_t k = S[p];
            double u = 0.0;
            for (int64_t j = 0; j < d; j++) u += ld(x, x_dt, t * d + j) * ld(w_up, w_dt, j * d_ff + k);
            h[p] = g[t * d_ff + k] * u;
            if (u_out) u_out[t * d_ff + k] = u;
        }
        if (u_out)
            for (int64_t k = 0, p = 0; k < d_ff; k++) {
                if (p < m && S[p] == k) { p++; continue; }
                u_out[t * d_ff + k] = 0.0;
            }
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < d; j++) {
            double acc = 0.0;
            for (int32_t p = 0; p < m; p++) acc += h[p] * ld(w_down, w_dt, (int64_t)S[p] * d + j);
            y[t * d + j] = acc;
        }
    }
    free(h);
}

/* Dense FFN: every channel, g given densely (0 off S_t), same ascending order:
 *   u = x W_up (all d_ff),  y[t,:] = sum_{k ascending} (g[t,k] u[t,k]) W_down[k,:] */
void oracle_dense_ffn(const void* x, int x_dt, const void* w_up, const void* w_down, int w_dt,
                      int64_t n, int64_t d, int64_t d_ff, const double* g, double* y) {
    double* u = (double*)malloc(sizeof(double) * (size_t)(n * d_ff > 0 ? n * d_ff : 1));
    oracle_vecmat(x, x_dt, w_up, w_dt, n, d, d_ff, u);
    for (int64_t t = 0; t < n; t++) {
        for (int64_t k = 0; k < d_ff; k++) u[t * d_ff + k] *= g[t * d_ff + k];
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < d; j++) {
            double acc = 0.0;
            for (int64_t k = 0; k < d_ff; k++) acc += u[t * d_ff + k] * ld(w_down, w_dt, k * d + j);
            y[t * d + j] = acc;
        }
    }
    free(u);
}
