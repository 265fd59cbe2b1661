/*
 * sketchssm.h -- C ABI of the SketchSSM decode path on NVIDIA B200 (sm_100a).
 *
 * SketchSSM ("Write to the Full State, Read from a Compact Sketch", arXiv
 * 2609.33051) keeps exact updates of a linear-attention / SSM recurrent state
 * but, between periodic flushes, answers reads from a low-rank sketch of it:
 *
 *   - state update  S_t = M_t S_{t-1} + B_t, read o_t = S_t^T q_t
 *       (SketchSSM project page, "01 / The idea", equation "Full state");
 *   - flush, once per window of W steps: read the full state once, apply the
 *       W buffered updates, write it back and refresh the sketch
 *       U = S^T Omega (project page, "02 / How to Make a Sketch"; paper §4.1
 *       and App. B as summarised on the paperlayer page);
 *   - non-flush steps: o^ = U (C q~) + (exact term of the buffered updates),
 *       with q~ the query mapped back through the buffered transitions
 *       (project page, "Coefficient vector & readout"; paper §3.2, §C.1).
 *
 * Families (B_t = b_t k_t v_t^T in all three):
 *   SS_MAMBA2  M_t = a_t I,                          a_t = exp(dt_t A_h), b_t = dt_t
 *   SS_GDN     M_t = a_t (I - beta_t k_t k_t^T),      b_t = beta_t
 *   SS_KDA     M_t = (I - beta_t k_t k_t^T) Diag(a_t), a_t in (0,1)^dk, b_t = beta_t
 *
 * Conventions for every entry point:
 *   - Ownership: the caller allocates every device buffer; the library keeps
 *     only a small host-side plan (shapes, ranks, window phase).  No call
 *     allocates device memory or synchronises the stream.
 *   - Pointers marked "device" must be device (or managed) addresses aligned
 *     to 16 bytes; a misaligned pointer returns SS_ERR_ALIGNMENT.
 *   - Launches are asynchronous on `stream` (NULL = the legacy default
 *     stream).  A call rejected by its checks (any status but SS_ERR_CUDA)
 *     launches nothing and leaves the plan unchanged.  SS_ERR_CUDA means a
 *     kernel launch failed: kernels the call queued before it stay queued and
 *     the plan accounts for them (a flush whose dense-head copies failed
 *     leaves the plan at phase 0 with no valid sketch, so ss_prime comes
 *     next).  Errors raised later by the device surface on the caller's next
 *     CUDA synchronisation.
 *   - No call throws, exits or aborts; every call returns an ss_status.
 *     ss_last_error_string() describes the last failure on this thread.
 *   - bf16 tensors are passed as their uint16_t bit patterns.
 *
 * Layouts (row-major, B = batch, H = heads, R = sum of ranks):
 *   state      float    [B][H][dk][dv]        device, read/write
 *   ring_k     uint16_t [B][H][W][dk]  bf16   device, read/write
 *   ring_v     uint16_t [B][H][W][dv]  bf16   device, read/write
 *   ring_gate  float    [B][H][Wg]            Mamba-2 dt / GDN a  (Wg = W rounded up to 4)
 *              float    [B][H][W][dk]         KDA a
 *   ring_beta  float    [B][H][Wg]            GDN/KDA beta; unused for Mamba-2 (may be NULL)
 *   sketch     float or bf16 [B][R][dv]       row off_h + i is u_i = S^T omega_i of head h
 *   basis      float    [R][dk]               row off_h + i is omega_i of head h (shared by the batch)
 *   coef       float    [R][dk]               rows off_h .. off_h + r_h - 1 are head h's map C
 *   coef_state float or bf16 [B][R][dk]       SS_COEF_STATE, SS_COEF_LRD: sequence b's map rows of head h at
 *                                             off_h .. off_h + r_h - 1 (dtype of the sketch)
 *   A          float    [H]                   Mamba-2 decay rates (A_h < 0 for decay)
 *   q, k       uint16_t [B][H][dk] bf16;  v uint16_t [B][H][dv] bf16
 *   gate       float    [B][H] (Mamba-2 dt, GDN a) or [B][H][dk] (KDA a)
 *   beta       float    [B][H] (GDN/KDA)
 *   out        float    [B][H][dv]
 *   with off_h = r_0 + ... + r_{h-1}.
 */
#ifndef SKETCHSSM_H
#define SKETCHSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st* ss_stream;

typedef enum {
    SS_OK = 0,
    SS_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, unknown enum */
    SS_ERR_ALIGNMENT = 2,     /* a device pointer is not 16-byte aligned */
    SS_ERR_UNSUPPORTED = 3,   /* shape outside the compiled set */
    SS_ERR_SCHEDULE = 4,      /* call not legal at the plan's window phase */
    SS_ERR_CUDA = 5           /* the CUDA runtime refused the launch */
} ss_status;

typedef enum { SS_MAMBA2 = 0, SS_GDN = 1, SS_KDA = 2 } ss_family;
typedef enum { SS_F32 = 0, SS_BF16 = 1 } ss_sketch_dtype;

/* Supported sizes: dk, dv in {64, 128}; 1 <= window <= 32; 1 <= heads <=
 * SS_MAX_HEADS; batch >= 1; 0 <= ranks[h] <= dk. */
#define SS_MAX_HEADS 512
#define SS_MAX_WINDOW 32

/* Bits a kernel ORs into ss_buffers.status (a device word the caller owns
 * and clears).  Kernels that wait for their own bulk copies bound each wait
 * to about one second; if a wait runs out the kernel sets SS_DEVICE_TIMEOUT
 * and returns without completing its outputs. */
#define SS_DEVICE_TIMEOUT 1
/* Set by ss_step_mixed when a fill count lies outside 0..W-1: that sequence
 * is neither decoded nor flushed and its fill_out entry is left as it was. */
#define SS_DEVICE_BAD_FILL 2
/* Set by a flush in SS_COEF_STATE or SS_COEF_LRD mode when a head's Gram matrix
 * (U^T U + lambda I, or P^T H P + lambda I) is not numerically positive definite (a Cholesky pivot
 * <= 0 or not finite, e.g. an all-zero state with rho = 0): that head's map
 * rows are written as zeros. */
#define SS_DEVICE_SINGULAR_MAP 4

/* Which coefficient map the non-flush read c = C q~ uses (project page,
 * "Per step · Non-flush: Coefficient vector & readout"). */
typedef enum {
    SS_COEF_FIXED = 0,       /* C = bufs->coef: one fp32 [R][dk] map shared by the batch */
    SS_COEF_STATE = 1,       /* per (sequence, head) map C = (U^T U + lambda I)^-1 U^T S^T,
                              * lambda = rho tr(U^T U) / r (project page, "Per window ·
                              * Flush: Sketch & coefficient map"; paper §A.2.1), rebuilt
                              * by every flush from the new state and sketch, fused into
                              * it (no second state read); stored in bufs->coef_state */
    SS_COEF_LRD = 2          /* per (sequence, head) map of the low-rank-plus-diagonal
                              * state metric (paper §A.2.2): H = L L^T + D, L = the 4
                              * output columns of the new state S with the largest
                              * energy ||S[:, v]||^2 (the lower column on a tie), D =
                              * the diagonal of the other columns' contribution;
                              * C = (P^T H P + lambda I)^-1 P^T H with the head's basis
                              * P, lambda = rho tr(P^T H P) / r.  Built, stored and read
                              * like SS_COEF_STATE (same buffers and layout); needs
                              * room for the pivots and the r x r Gram matrix in the
                              * flush's tile buffer (ss_create returns
                              * SS_ERR_UNSUPPORTED for a rank beyond it) */
} ss_coef_mode;

typedef struct {
    int32_t family;          /* ss_family */
    int32_t batch;           /* B: sequences decoded together */
    int32_t heads;           /* H: state heads per sequence */
    int32_t dk;              /* key / query dimension = state rows (Mamba-2 dstate) */
    int32_t dv;              /* value dimension = state columns (Mamba-2 headdim) */
    int32_t window;          /* W: steps per flush window */
    const int32_t* ranks;    /* host [heads]: sketch rank r_h of each head; copied */
    int32_t sketch_dtype;    /* ss_sketch_dtype of the stored sketch U */
    int32_t coef_mode;       /* ss_coef_mode; 0 (zero-initialised) = SS_COEF_FIXED */
    float coef_ridge;        /* rho >= 0 of SS_COEF_STATE and SS_COEF_LRD (else ignored) */
    const uint8_t* dense_heads; /* host [heads] or NULL; copied.  Nonzero: a dense-fallback head
                              * (paper App. D: at non-flush steps it reads a BF16 copy of its
                              * state).  Its rank must be dk; its dk sketch rows hold the
                              * copy, row k = S[k][:] in the sketch dtype, written by every
                              * flush with a sketch; its non-flush read is S0^T q~ + (buffered
                              * term), exact up to the copy's rounding.  Its basis, coef and
                              * coef_state rows are not read. */
} ss_config;

typedef struct ss_plan ss_plan;

typedef struct {
    size_t state, ring_k, ring_v, ring_gate, ring_beta, sketch, basis, coef, A;
    size_t q, k, v, gate, beta, out;
    size_t coef_state;       /* SS_COEF_STATE, SS_COEF_LRD: [B][R][dk] in the sketch dtype; else 0 */
    int32_t total_rank;      /* R = sum of ranks */
    int32_t gate_stride;     /* Wg (scalar-gate families) or W * dk (KDA), floats per (b, h) */
} ss_sizes;

typedef struct {
    float* state;            /* device, see layouts */
    uint16_t* ring_k;
    uint16_t* ring_v;
    float* ring_gate;
    float* ring_beta;        /* may be NULL for Mamba-2 */
    void* sketch;            /* NULL: no sketch is kept (ReplaySSM flushes) */
    const float* basis;      /* needed when sketch != NULL */
    const float* coef;       /* needed by ss_decode_step */
    const float* A;          /* needed for Mamba-2 */
    int32_t* status;         /* optional device int32 (4-byte aligned), see SS_DEVICE_TIMEOUT; NULL: no report */
    void* coef_state;        /* SS_COEF_STATE and SS_COEF_LRD only: device [B][R][dk] in the sketch dtype, the
                              * per-(sequence, head) maps (head h's rows at the rank offset,
                              * like the sketch); written by ss_prime / ss_flush with a sketch,
                              * read by ss_decode_step; bufs->coef is then unused */
} ss_buffers;

typedef struct {
    const uint16_t* q;       /* device bf16 [B][H][dk] */
    const uint16_t* k;       /* device bf16 [B][H][dk] */
    const uint16_t* v;       /* device bf16 [B][H][dv] */
    const float* gate;       /* device [B][H] or KDA [B][H][dk] */
    const float* beta;       /* device [B][H]; may be NULL for Mamba-2 */
    float* out;              /* device [B][H][dv] */
} ss_step_io;

/* Operation codes for ss_traffic_bytes. */
typedef enum {
    SS_OP_DECODE = 0,        /* ss_decode_step at phase tau */
    SS_OP_FLUSH = 1,         /* ss_flush with a token at phase W-1 (tau ignored) */
    SS_OP_FLUSH_NO_TOKEN = 2,/* ss_flush(io = NULL) at phase tau */
    SS_OP_PRIME = 3,         /* ss_prime */
    SS_OP_EXACT = 4,         /* ss_exact_step */
    SS_OP_REPLAY = 5,        /* ss_replay_step at phase tau */
    SS_OP_REPLAY_FLUSH = 6   /* ss_flush with a token and sketch == NULL */
} ss_op;

typedef struct {
    /* State-access traffic as the paper counts it (paper App. D, Table 4 as
     * summarised on the paperlayer page): fp32 state reads and writes plus
     * bf16 sketch + coefficient-map reads of G (dk + dv) elements per head at
     * non-flush steps (plus G W bf16 projected erase vectors for GDN/KDA); a
     * dense-fallback head reads a bf16 dk x dv state copy instead.
     * Ring-buffer traffic and sketch/map writes are excluded, as there. */
    double paper_read_bytes;
    double paper_write_bytes;
    /* Every byte this library's kernels for the call must move (inputs,
     * ring slots, state, sketch, basis/map once per head or per sequence,
     * outputs, and the extra state read that writes dense heads' copies).
     * This is the numerator of the HBM roofline. */
    double read_bytes;
    double write_bytes;
} ss_traffic;

/* Create a plan for one layer's decode.  The config (and ranks) are copied.
 * Returns SS_ERR_INVALID_ARG / SS_ERR_UNSUPPORTED for bad shapes.
 * SS_ERR_UNSUPPORTED also when a call of the plan would need more shared
 * memory than one CTA has: the flush stages the window's keys, values and
 * decays plus the basis rows of one head, and the decode step stages, per
 * warp, the window's ring slots and sketch rows plus the head's map C
 * (rmax x dk fp32), so very large ranks with long windows may not fit (KDA
 * with rank 128, dk = dv = 128 and W = 32 does not).  Every rank up to 64 at W <= 16,
 * and up to 32 at W <= 32, is supported.  SS_COEF_STATE needs every rank
 * <= dv (U^T U must be invertible) and a finite coef_ridge >= 0; its flushes
 * run on the CUDA-core flush kernel for every family.  SS_COEF_LRD likewise,
 * with every rank small enough for its scratch: up to 56 at dk = dv = 64,
 * 64 at dk = 64, dv = 128, 81 at dk = 128, dv = 64 and 118 at dk = dv = 128.  The plan starts at
 * phase 0 with no valid sketch. */
ss_status ss_create(const ss_config* cfg, ss_plan** out);
ss_status ss_destroy(ss_plan* plan);

/* Bytes of every buffer the caller must allocate for this plan. */
ss_status ss_buffer_sizes(const ss_plan* plan, ss_sizes* out);

/* Window phase (tokens buffered since the last flush) and whether the
 * sketch is current.  ss_set_phase restores both, e.g. from a checkpoint of
 * (state, ring, sketch); 0 <= phase <= W-1. */
ss_status ss_get_phase(const ss_plan* plan, int32_t* phase, int32_t* sketch_valid);
ss_status ss_set_phase(ss_plan* plan, int32_t phase, int32_t sketch_valid);

/* U = S^T Omega from the current state with nothing buffered: a flush of
 * zero updates (project page, "Precompute the basis outputs").  Legal at
 * phase 0; needs bufs->sketch and bufs->basis.  Marks the sketch valid. */
ss_status ss_prime(ss_plan* plan, const ss_buffers* bufs, ss_stream stream);

/* Non-flush step (project page, "Per step · Non-flush"; paper §3.2, §C.1).
 * Legal at phase p in 0..W-2 with a valid sketch.  Appends this token to
 * ring slot p, then writes
 *     out = U (C q~) + sum_{j<=p} b_j (k_j . x_j) v_j,
 * x_p = q, x_{j-1} = M_j^T x_j, q~ = x_{-1}, without reading the state.
 * Phase becomes p+1. */
ss_status ss_decode_step(ss_plan* plan, const ss_buffers* bufs, const ss_step_io* io,
                         ss_stream stream);

/* Flush (paper §4.1, App. B).  With io != NULL: legal at phase W-1; the token
 * is the window's W-th update; reads the state once, applies the W updates in
 * order, writes the state, writes out = S_W^T q, and, if bufs->sketch !=
 * NULL, refreshes U = S_W^T Omega (the sketch is then valid; otherwise it is
 * marked stale).  With io == NULL: legal at any phase tau; applies the tau
 * buffered updates, writes the state and (if bufs->sketch) the sketch; no
 * output.  Phase becomes 0.  The ring slots are not modified. */
ss_status ss_flush(ss_plan* plan, const ss_buffers* bufs, const ss_step_io* io,
                   ss_stream stream);

/* Standard baseline: S <- M S + B, out = S^T q, every step (paper App. D,
 * "Standard").  Legal at phase 0; marks the sketch stale. */
ss_status ss_exact_step(ss_plan* plan, const ss_buffers* bufs, const ss_step_io* io,
                        ss_stream stream);

/* ReplaySSM baseline non-flush step (GitHub repository page, "Overview";
 * paper §1-§2): appends the token at slot p like ss_decode_step and writes
 * the exact out = S0^T q~ + (buffered term), reading the full state but not
 * writing it.  Legal at phase 0..W-2; phase becomes p+1.  Its flush is
 * ss_flush with bufs->sketch == NULL. */
ss_status ss_replay_step(ss_plan* plan, const ss_buffers* bufs, const ss_step_io* io,
                         ss_stream stream);

/* One step of a batch whose sequences sit at different window positions
 * (project page, "Per step"; paper §3.2 and §4.1 applied per sequence).
 * fill_in[b] (device int32[batch], 4-byte aligned) is the number of tokens
 * sequence b has buffered since its last flush, 0..W-1.  Sequences with
 * fill_in[b] <= W-2 take the non-flush step of ss_decode_step at their own
 * slot fill_in[b]; sequences with fill_in[b] == W-1 take ss_flush with this
 * token and refresh their sketch rows.  fill_out[b] (device int32[batch],
 * must not alias fill_in) receives (fill_in[b] + 1) mod W.  A value outside
 * 0..W-1 sets SS_DEVICE_BAD_FILL in bufs->status; that sequence's outputs,
 * ring, state and fill_out entry are left as they were.  Needs the plan at
 * phase 0 with a valid sketch (ss_prime), bufs->state, sketch, basis, coef
 * (and A for Mamba-2); the plan's phase is not used and stays 0.  The
 * decode runs on `stream`; the flush runs beside it on a stream the plan
 * owns (created on first use), forked from `stream` after its earlier work
 * and joined back to it with events, so work queued on `stream` afterwards
 * sees both (this also holds under stream capture).  If a launch fails
 * after the fork, the side stream is still joined back before the error
 * (SS_ERR_CUDA) is returned.  The fills are read on the device only. */
ss_status ss_step_mixed(ss_plan* plan, const ss_buffers* bufs, const ss_step_io* io,
                        const int32_t* fill_in, int32_t* fill_out, ss_stream stream);

/* Traffic of one call for the whole batch (see ss_traffic).  tau = phase
 * before the call for SS_OP_DECODE / SS_OP_REPLAY / SS_OP_FLUSH_NO_TOKEN. */
ss_status ss_traffic_bytes(const ss_plan* plan, int32_t op, int32_t tau, ss_traffic* out);

/* Number of kernels this library has launched in this process. */
uint64_t ss_launch_count(void);

/* Testing hook.  With stall != 0 the next launching call of this plan
 * (ss_prime, ss_decode_step, ss_flush, ss_exact_step or ss_replay_step)
 * makes one CTA expect more bytes than its bulk copies deliver, so
 * that CTA's bounded wait runs out after about a second: it sets
 * SS_DEVICE_TIMEOUT in bufs->status and returns, leaving its outputs
 * incomplete; the rest of the launch completes.  The hook clears itself
 * after that call.  Used to test the timeout path without a device fault. */
ss_status ss_debug_stall_next_copy(ss_plan* plan, int32_t stall);

/* Testing hook for the host-side launch-failure paths.  With n > 0, the
 * n-th kernel launch that this plan's calls make from now on (counting
 * every launch of every call: a flush with dense heads makes two, a mixed
 * step two or three) is not made: the call behaves as if the CUDA runtime
 * had refused it (SS_ERR_CUDA, "injected launch failure").  Launches queued
 * before it stay queued and the plan accounts for them, as for a real
 * failure.  The hook clears itself when it fires; n = 0 disarms it.  No
 * device code is involved, so the path is tested without a GPU fault. */
ss_status ss_debug_fail_launch(ss_plan* plan, int32_t n);

const char* ss_status_string(ss_status status);
const char* ss_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* SKETCHSSM_H */
