/*
 * sffn -- activation-sparse gated FFN inference on one B200 (sm_100a).
 *
 * Computes, for n tokens x (n x d),
 *
 *     z = x W_gate                       (dense gate, d x d_ff)
 *       or  z = (x A) B                  (LoPA low-rank gate, A d x r, B r x d_ff)
 *     S_t = { k : z[t,k] > tau }         threshold select, g = z - tau on S_t
 *       or  the K largest SiLU(z[t,k])   per-token top-K select, g = SiLU(z) on S_t
 *     y[t,:] = sum_{k in S_t} g[t,k] <x[t,:], W_up[:,k]> W_down[k,:]
 *
 * "Model Casting and Low-Parameter Gating: Towards More Sparsely Activated
 * FFNs" (abstract): compute the gating matrix's output first and, because its
 * activation is highly sparse, skip the two other matrices for the inactive
 * channels; LoPA gives the gate fewer parameters and FLOPs than the other two
 * matrices.  "Mixture-of-Channels" (sections "Dentro il mixture", "Dentro
 * MoC"): keep per token only the top-K channels ranked by the SwiGLU gate and
 * load only those channels' weight rows.
 *
 * Conventions for every entry point:
 *  - Return 0 (SFFN_OK) or a positive sffn_status code; nothing aborts.
 *  - A `stream` argument is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Calls that take a stream are asynchronous on it unless
 *    stated otherwise.
 *  - Device pointers must be 16-byte aligned and on the handle's device.
 *  - A handle is not thread-safe: one host thread at a time, and forwards on
 *    one handle must be ordered (same stream, or the caller orders them),
 *    because they share the handle's workspace.
 *  - Device-side failures are recorded, not trapped.  Every wait inside a
 *    kernel (on a bulk copy, a tensor-core commit, a grid barrier or another
 *    CTA's part) is bounded in time; a wait that runs out sets the timeout bit
 *    of the handle's sticky status word and the kernel returns early.  The down
 *    kernel checks the channel ids and counts it reads from the gate kernel's
 *    lists and skips any that lie outside their segment, setting the bounds
 *    bit.  The word is mirrored into host-mapped memory, so sffn_forward,
 *    sffn_forward_dense and sffn_forward_host return SFFN_ERR_TIMEOUT or
 *    SFFN_ERR_DEVICE_CHECK, and launch nothing, once a forward that failed has
 *    finished on the device.  The word stays set for the handle's lifetime:
 *    destroy the handle and make a new one.
 */
#ifndef SFFN_H
#define SFFN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sffn_ctx* sffn_handle;

typedef enum {
    SFFN_OK = 0,
    SFFN_ERR_INVALID_ARG = 1,  /* NULL or misaligned pointer, bad size, NaN tau, ... */
    SFFN_ERR_NOT_READY = 2,    /* forward before sffn_set_weights */
    SFFN_ERR_UNSUPPORTED = 3,  /* e.g. LoPA forward on a handle without A and B */
    SFFN_ERR_CUDA = 4,         /* a CUDA runtime call or a launch failed */
    SFFN_ERR_OOM = 5,          /* device allocation failed */
    SFFN_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out (sticky) */
    SFFN_ERR_DEVICE_CHECK = 7  /* a kernel's own bounds check failed (sticky) */
} sffn_status;

typedef enum { SFFN_BF16 = 0, SFFN_F32 = 1 } sffn_dtype;
typedef enum { SFFN_GATE_DENSE = 0, SFFN_GATE_LOPA = 1 } sffn_gate_mode;
typedef enum { SFFN_SELECT_THRESHOLD = 0, SFFN_SELECT_TOPK = 1, SFFN_SELECT_TOPP = 2 } sffn_select_kind;

/* Model shape.  d and lopa_rank must be multiples of 8 (16-byte weight rows);
 * lopa_rank = 0 means no LoPA gate; 1 <= max_tokens <= 1024; wdtype is the
 * storage type of weights, x and y (bf16, or fp32 for small exact checks);
 * device is the CUDA ordinal. */
typedef struct {
    int32_t d;
    int32_t d_ff;
    int32_t lopa_rank;
    int32_t max_tokens;
    int32_t wdtype;      /* sffn_dtype */
    int32_t device;
} sffn_config;

/* Channel selection.  THRESHOLD: active iff z > tau, activation z - tau (a
 * shifted ReLU); tau = +inf selects nothing, NaN or -inf is rejected.
 * TOPK: per token the k channels with the largest SiLU(z) (ties to the lower
 * channel index), activation SiLU(z); 0 <= k <= d_ff.
 * TOPP ("PrunePath", abstract: a softmax-normalised routing distribution with
 * a cumulative-mass threshold): per token the shortest run of channels by
 * descending z (ties to the lower index) whose softmax mass reaches p,
 * activation SiLU(z); 0 <= p <= 1 (0 selects nothing).  The masses are summed
 * as integers, exp(z - max z) in units of 2^-S with d_ff 2^S < 2^30, so the
 * choice is reproducible; it can differ from the exact one only where the
 * cumulative mass lies within that rounding of the budget. */
typedef struct {
    int32_t kind;        /* sffn_select_kind */
    float tau;           /* THRESHOLD */
    int32_t k;           /* TOPK */
    float p;             /* TOPP */
} sffn_select;

/* Allocate a handle and its device workspace, sized for cfg->max_tokens,
 * plus one small host-mapped pinned block (the status mirror).
 * The library owns all memory it allocates; sffn_destroy frees it.
 * Errors: INVALID_ARG (bad shape), CUDA (bad device), OOM; on any error
 * nothing stays allocated and *out is NULL.
 * Failure testing: with the environment variable SFFN_FAULT set to "alloc:N"
 * (or "copy:N") the N-th allocation (or host-to-device copy) made by one call
 * of sffn_create or sffn_set_weights reports failure without being made. */
int sffn_create(sffn_handle* out, const sffn_config* cfg);

/* Copy the weights in (host or device memory, src_is_device says which) and
 * repack them channel-major into library-owned buffers, so that channel k of
 * W_gate, W_up and B, and row k of W_down, are each one contiguous row.
 * Inputs are row-major in the handle's wdtype:
 *   w_gate d x d_ff,  A d x r,  B r x d_ff,  w_up d x d_ff,  w_down d_ff x d.
 * w_gate may be NULL when A and B are given and vice versa (not all three
 * NULL); A and B need lopa_rank > 0.  The caller keeps ownership of its
 * buffers.  Synchronises `stream` before returning.
 * Errors: INVALID_ARG, CUDA, OOM; after an error the handle holds no weights
 * (NOT_READY) and nothing it allocated for them stays allocated. */
int sffn_set_weights(sffn_handle h, const void* w_gate, const void* A, const void* B,
                     const void* w_up, const void* w_down, int src_is_device, void* stream);

/* Sparse forward.  x: n_tokens x d device buffer, out: n_tokens x d device
 * buffer, both in wdtype and caller-owned.  gate_mode: sffn_gate_mode.
 * Asynchronous on `stream`, no host synchronisation; n_tokens = 0 is a no-op.
 * The output is deterministic: the same inputs give bitwise the same y.
 * Errors: INVALID_ARG, NOT_READY, UNSUPPORTED, CUDA; TIMEOUT or DEVICE_CHECK
 * when an earlier forward on the handle recorded a device-side failure. */
int sffn_forward(sffn_handle h, const void* x, int n_tokens, int gate_mode,
                 const sffn_select* sel, void* out, void* stream);

/* The same library's dense FFN: every channel's W_gate, W_up and W_down row is
 * read and multiplied; the activation (and top-K mask) is the same, so y
 * equals the sparse forward's up to rounding.  Same arguments and errors. */
int sffn_forward_dense(sffn_handle h, const void* x, int n_tokens, int gate_mode,
                       const sffn_select* sel, void* out, void* stream);

/* sffn_forward with HOST buffers: copies x_host to the device, runs the
 * forward and delivers the result into out_host, all on `stream`, then
 * synchronises it.  Pinned host memory gives asynchronous copies.  With one or
 * two tokens, page-locked buffers that the device can address (memory from
 * cudaHostAlloc / cudaMallocHost or cudaHostRegister under unified
 * addressing) are read and written by the fused decode kernel itself: it
 * pulls x_host in at its start and stores y into out_host, so neither takes a
 * copy-engine round trip.  Errors: as sffn_forward. */
int sffn_forward_host(sffn_handle h, const void* x_host, int n_tokens, int gate_mode,
                      const sffn_select* sel, void* out_host, void* stream);

/* The last forward's active channels per token, for checking: idx (host,
 * n_tokens x d_ff int32) receives token t's ascending channel list at row t,
 * counts (host, n_tokens) its length, *union_size (host, may be NULL) the
 * number of distinct channels over all tokens.  The lists are the kernels'
 * own decisions: the fused decode kernel's compacted lists, the tensor-core
 * gate's per-token selection bits (threshold), or the selection kernel's
 * masks (top-K, top-p).  Synchronises the last forward's stream.
 * Errors: INVALID_ARG, NOT_READY (no forward yet), CUDA, and the status
 * word's TIMEOUT or DEVICE_CHECK. */
int sffn_get_active(sffn_handle h, int32_t* idx, int32_t* counts, int32_t* union_size);

/* The union bitmap the last tensor-core forward's up and down kernels took
 * their active 128-channel blocks from (bit k of word k / 32: some token of
 * the pass selected channel k; for more than 128 tokens, the last pass of
 * 128).  bits: host, nwords >= ceil(d_ff / 32) words (words past that are
 * zeroed).  Synchronises the last forward's stream.  Errors: INVALID_ARG,
 * NOT_READY, UNSUPPORTED (the last forward did not take the tensor-core
 * path), CUDA, and the status word's TIMEOUT or DEVICE_CHECK. */
int sffn_get_union(sffn_handle h, uint32_t* bits, int nwords);

/* Heavy-hitter channels (the heavy-hitter split, an abstract in the "FFN
 * modules" paper listing: a few FFN neurons carry a large output for every
 * input while the rest fire sparsely, so the FFN is split into a part for
 * those neurons and a sparse rest).  `channels` (host, `count` entries, each
 * in [0, d_ff), duplicates allowed, NULL when count = 0) names the hot
 * channels; count = 0 clears the set.  With a set, the fused decode kernel
 * (threshold selection, one or two tokens) reads every hot channel's W_up
 * row and takes its up dot products when the forward starts, alongside the
 * gate stream rather than after the gate has selected the channel, and uses
 * them for the hot channels the gate selects; the other channels stay
 * gate-first.  Selection and activation are unchanged, so y and the active
 * lists are bitwise those of the same forward without a hot set (a hot
 * channel the gate does not select contributes nothing); the set changes
 * which bytes are read and when.  Other paths ignore it.  Synchronous.
 * Errors: INVALID_ARG (count < 0, channels NULL with count > 0, a channel
 * outside [0, d_ff)), CUDA. */
int sffn_set_hot(sffn_handle h, const int32_t* channels, int count);

/* Record timing events around each kernel of later forwards (profiling):
 * events[0] before the first launch and events[i] after launch i; at most
 * n_events events are recorded (cudaEvent_t passed as void*, created by the
 * caller and kept alive while set).  n_events = 0 switches recording off.
 * sffn_last_launches stores in *launches the number of kernels the last
 * forward launched.  Errors: INVALID_ARG. */
int sffn_set_stage_events(sffn_handle h, void* const* events, int n_events);
int sffn_last_launches(sffn_handle h, int32_t* launches);

/* Name of kernel i (0-based, launch order) of the last forward, for
 * profiles and timing reports; "" when there is no such kernel. */
const char* sffn_last_kernel_name(sffn_handle h, int i);

/* Synchronise the device and read the handle's sticky device status word
 * (see the conventions above).  Returns SFFN_OK, SFFN_ERR_DEVICE_CHECK (a
 * bounds check failed), or SFFN_ERR_TIMEOUT (a bounded wait ran out); the
 * word stays set.  Also INVALID_ARG, CUDA. */
int sffn_check_status(sffn_handle h);

/* Failure testing: arm a one-shot, host-side injection on the handle.
 *  SFFN_INJECT_WAIT_TIMEOUT, arg = a wait limit in ns (1e3 .. 2e9): the next
 *    fused decode forward (threshold selection, one or two tokens) waits at
 *    its final grid barrier for one arrival more than the grid makes, gives up
 *    after `arg` ns, records the timeout and leaves y unwritten; later calls
 *    return SFFN_ERR_TIMEOUT.
 *  SFFN_INJECT_BAD_LIST_ENTRY: the next forward that runs the separate down
 *    kernel (fp32 top-K, for instance) has the host overwrite, between the
 *    gate and the down kernel, the first entry of the first list segment with
 *    a channel outside every segment and the second segment's count with one
 *    beyond its slots; the down kernel's checks skip both and record them;
 *    later calls return SFFN_ERR_DEVICE_CHECK.
 * Nothing here makes a kernel fault: the failures are planted by the host and
 * caught by the kernels' own bounded waits and checks.  Errors: INVALID_ARG. */
enum { SFFN_INJECT_WAIT_TIMEOUT = 1, SFFN_INJECT_BAD_LIST_ENTRY = 2 };
int sffn_debug_inject(sffn_handle h, int what, long long arg);

/* Sparse forward that allocates no device memory, for callers that cannot
 * call cudaMalloc while they run: a host runtime that owns all device memory
 * through its own pool, or latency-critical code where an allocation (which
 * can synchronise the device) is not allowed after start-up.  No handle is
 * used (creating one allocates); the weights come from the caller.  The
 * pages describe no such interface: this entry point has no counterpart in
 * them.
 *
 * Computes the dense-gate, threshold-select forward of sffn_forward:
 * y[t,:] = sum_{k: z[t,k] > tau} (z[t,k] - tau) <x[t,:], W_up[:,k]> W_down[k,:].
 * Inputs are device buffers in `wdtype` (SFFN_BF16 or SFFN_F32), 16-byte
 * aligned, on the current device, owned by the caller:
 *   w_gate_cm  d_ff x d   row k is column k of W_gate
 *   w_up_cm    d_ff x d   row k is column k of W_up
 *   w_down     d_ff x d   W_down as is
 *   x          n_tokens x d;   out  n_tokens x d
 * Limits: d a multiple of 8 and <= 8192, 1 <= d_ff <= 32768,
 * 0 <= n_tokens <= 8; beyond them the call returns SFFN_ERR_INVALID_ARG and
 * prints why.  tau: a number or +inf.
 * Scratch: one file-scope device array of about 3.9 MiB, reserved on every GPU
 * that loads the library until the process exits.  Every call shares it and
 * it keeps the last call's contents (the call clears what must start at
 * zero), so calls whose kernels overlap on the GPU -- on two streams, or from
 * two threads -- race and give wrong results: order them.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, once per
 * device); make that first call before any stream capture.
 * Device-side failures (a bounded wait that ran out, a list entry the down
 * kernel's checks rejected) set a status word inside the scratch, which stays
 * set until sffn_noalloc_check_status reads it.
 * Asynchronous on `stream` (cudaStream_t as void*, NULL = legacy default).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int sffn_forward_noalloc(const void* w_gate_cm, const void* w_up_cm, const void* w_down, int d, int d_ff,
                         int wdtype, const void* x, int n_tokens, float tau, void* out, void* stream);

/* Synchronise the current device and read, then clear, the status word that
 * sffn_forward_noalloc's kernels set on this device.  Returns SFFN_OK (also
 * when no such call has run on the device), SFFN_ERR_TIMEOUT or
 * SFFN_ERR_DEVICE_CHECK (some call since the last read failed: its output is
 * not to be trusted), or SFFN_ERR_CUDA.  Allocates nothing. */
int sffn_noalloc_check_status(void);

/* Free the handle and everything it owns.  NULL is accepted. */
int sffn_destroy(sffn_handle h);

/* Static description of a status code (never NULL). */
const char* sffn_strerror(int code);

/* Detail of the calling thread's most recent failure (never NULL; "" if none). */
const char* sffn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SFFN_H */
