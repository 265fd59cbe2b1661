// Host side of the SketchSSM C ABI (include/sketchssm.h): plans, argument
// and schedule validation, the traffic model and kernel dispatch.  No call
// here allocates device memory or synchronises a stream.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "ss_internal.h"

namespace ss {
int flush_smem_bytes(int family, int dk, int dv, int n, int rpad, bool smap);
int decode_smem_bytes(int family, int dk, int dv, int P, int rmax, int esz, bool smap, bool dense_any);
bool flush_map_fits(int dk, int dv, int r);
bool flush_lrd_fits(int dk, int dv, int r);
}  // namespace ss

struct ss_plan {
    ss_config cfg;
    int32_t ranks[SS_MAX_HEADS];
    int32_t off[SS_MAX_HEADS + 1];
    int32_t R, rmax, Wg;      // rmax: largest rank of a sketched (not dense) head
    uint32_t dense[SS_MAX_HEADS / 32];
    int32_t n_dense;
    // ss_step_mixed runs its flush on a second stream beside the decode,
    // forked from and joined back to the caller's stream (created on first use).
    cudaStream_t side;
    cudaEvent_t fork, join;
    int32_t phase;
    int32_t sketch_valid;
    int32_t stall_next;
    int32_t fail_launch;      // testing hook: the launch (1-based, counted from arming) to refuse
};

namespace {

thread_local std::string g_err;
std::atomic<uint64_t> g_launches{0};
constexpr int kSmemLimit = 227 * 1024;

ss_status fail(ss_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

ss_status ok() {
    g_err.clear();
    return SS_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

#define REQUIRE_PTR(ptr, what)                                                     \
    do {                                                                           \
        if ((ptr) == nullptr) return fail(SS_ERR_INVALID_ARG, "%s is NULL", what); \
        if (!aligned16(ptr))                                                       \
            return fail(SS_ERR_ALIGNMENT, "%s is not 16-byte aligned", what);      \
    } while (0)

#define CHECK(expr)                       \
    do {                                  \
        const ss_status _s = (expr);      \
        if (_s != SS_OK) return _s;       \
    } while (0)

ss_status check_status(const ss_buffers* b) {
    if (b->status != nullptr && (reinterpret_cast<uintptr_t>(b->status) & 3u) != 0)
        return fail(SS_ERR_ALIGNMENT, "bufs->status is not 4-byte aligned");
    return SS_OK;
}

bool state_map(const ss_plan* pl) { return pl->cfg.coef_mode == SS_COEF_STATE || pl->cfg.coef_mode == SS_COEF_LRD; }

// The map buffer a flush that refreshes the sketch must also refresh.
ss_status check_map(const ss_plan* pl, const ss_buffers* b) {
    if (state_map(pl)) REQUIRE_PTR(b->coef_state, "bufs->coef_state");
    return SS_OK;
}

// Consume the testing hook: the stall applies to one launch only.
int take_stall(ss_plan* pl) {
    const int s = pl->stall_next;
    pl->stall_next = 0;
    return s;
}

ss_status check_ring(const ss_plan* pl, const ss_buffers* b) {
    REQUIRE_PTR(b->state, "bufs->state");
    REQUIRE_PTR(b->ring_k, "bufs->ring_k");
    REQUIRE_PTR(b->ring_v, "bufs->ring_v");
    REQUIRE_PTR(b->ring_gate, "bufs->ring_gate");
    if (pl->cfg.family != SS_MAMBA2) REQUIRE_PTR(b->ring_beta, "bufs->ring_beta");
    if (pl->cfg.family == SS_MAMBA2) REQUIRE_PTR(b->A, "bufs->A");
    return SS_OK;
}

ss_status check_io(const ss_plan* pl, const ss_step_io* io) {
    if (io == nullptr) return fail(SS_ERR_INVALID_ARG, "io is NULL");
    REQUIRE_PTR(io->q, "io->q");
    REQUIRE_PTR(io->k, "io->k");
    REQUIRE_PTR(io->v, "io->v");
    REQUIRE_PTR(io->gate, "io->gate");
    if (pl->cfg.family != SS_MAMBA2) REQUIRE_PTR(io->beta, "io->beta");
    REQUIRE_PTR(io->out, "io->out");
    return SS_OK;
}

ss::FlushParams flush_params(const ss_plan* pl, const ss_buffers* b, const ss_step_io* io) {
    ss::FlushParams p;
    std::memset(&p, 0, sizeof p);
    p.state = b->state;
    p.ring_k = b->ring_k;
    p.ring_v = b->ring_v;
    p.ring_gate = b->ring_gate;
    p.ring_beta = b->ring_beta;
    if (io) {
        p.tok_q = io->q; p.tok_k = io->k; p.tok_v = io->v;
        p.tok_gate = io->gate; p.tok_beta = io->beta; p.out = io->out;
    }
    p.sketch = b->sketch;
    p.basis = b->basis;
    p.A = b->A;
    p.status = b->status;
    p.B = pl->cfg.batch; p.H = pl->cfg.heads; p.W = pl->cfg.window; p.Wg = pl->Wg; p.R = pl->R;
    p.sketch_bf16 = pl->cfg.sketch_dtype == SS_BF16;
    if (state_map(pl) && b->sketch != nullptr) {
        p.cmap = b->coef_state;
        p.ridge = pl->cfg.coef_ridge;
        p.lrd = pl->cfg.coef_mode == SS_COEF_LRD;
    }
    std::memcpy(p.dense, pl->dense, sizeof p.dense);
    std::memcpy(p.off, pl->off, sizeof(int32_t) * (pl->cfg.heads + 1));
    return p;
}

ss::StepParams step_params(const ss_plan* pl, const ss_buffers* b, const ss_step_io* io) {
    ss::StepParams p;
    std::memset(&p, 0, sizeof p);
    p.state = b->state;
    p.ring_k = b->ring_k; p.ring_v = b->ring_v; p.ring_gate = b->ring_gate; p.ring_beta = b->ring_beta;
    p.tok_q = io->q; p.tok_k = io->k; p.tok_v = io->v; p.tok_gate = io->gate; p.tok_beta = io->beta;
    p.sketch = b->sketch; p.coef = b->coef; p.A = b->A; p.out = io->out; p.status = b->status;
    p.B = pl->cfg.batch; p.H = pl->cfg.heads; p.W = pl->cfg.window; p.Wg = pl->Wg; p.R = pl->R;
    p.p = pl->phase;
    p.sketch_bf16 = pl->cfg.sketch_dtype == SS_BF16;
    if (state_map(pl)) p.cmap = b->coef_state;
    std::memcpy(p.dense, pl->dense, sizeof p.dense);
    p.dense_any = pl->n_dense > 0;
    std::memcpy(p.off, pl->off, sizeof(int32_t) * (pl->cfg.heads + 1));
    return p;
}

ss_status launched(cudaError_t e, const char* what) {
    if (e != cudaSuccess)
        return fail(SS_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return SS_OK;
}

// Make one launch through the testing hook: when the plan's armed counter
// reaches this launch, the launch is not made and an error stands for it.
template <typename F>
ss_status launch_via(ss_plan* pl, const char* what, F&& fn) {
    if (pl->fail_launch > 0 && --pl->fail_launch == 0)
        return fail(SS_ERR_CUDA, "%s launch failed: injected launch failure", what);
    return launched(fn(), what);
}

int esize(const ss_plan* pl) { return pl->cfg.sketch_dtype == SS_BF16 ? 2 : 4; }

// After a flush that sketches: the dense-fallback heads' state copies.
ss_status dense_copies(ss_plan* pl, const ss::FlushParams& p, cudaStream_t st) {
    if (pl->n_dense == 0 || !p.do_sketch) return SS_OK;
    return launch_via(pl, "dense copy", [&] { return ss::launch_dense_copy(pl->cfg.dk, pl->cfg.dv, p, st); });
}

}  // namespace

extern "C" {

ss_status ss_create(const ss_config* cfg, ss_plan** out) {
    if (cfg == nullptr || out == nullptr) return fail(SS_ERR_INVALID_ARG, "cfg or out is NULL");
    *out = nullptr;
    const ss_config& c = *cfg;
    if (c.family < SS_MAMBA2 || c.family > SS_KDA) return fail(SS_ERR_INVALID_ARG, "unknown family %d", c.family);
    if (c.batch < 1) return fail(SS_ERR_INVALID_ARG, "batch %d < 1", c.batch);
    if (c.heads < 1 || c.heads > SS_MAX_HEADS)
        return fail(SS_ERR_UNSUPPORTED, "heads %d outside 1..%d", c.heads, SS_MAX_HEADS);
    if ((c.dk != 64 && c.dk != 128) || (c.dv != 64 && c.dv != 128))
        return fail(SS_ERR_UNSUPPORTED, "dk=%d dv=%d: supported sizes are 64 and 128", c.dk, c.dv);
    if (c.window < 1 || c.window > SS_MAX_WINDOW)
        return fail(SS_ERR_UNSUPPORTED, "window %d outside 1..%d", c.window, SS_MAX_WINDOW);
    if (c.sketch_dtype != SS_F32 && c.sketch_dtype != SS_BF16)
        return fail(SS_ERR_INVALID_ARG, "unknown sketch dtype %d", c.sketch_dtype);
    if (c.ranks == nullptr) return fail(SS_ERR_INVALID_ARG, "ranks is NULL");
    if (c.coef_mode != SS_COEF_FIXED && c.coef_mode != SS_COEF_STATE && c.coef_mode != SS_COEF_LRD)
        return fail(SS_ERR_INVALID_ARG, "unknown coef_mode %d", c.coef_mode);
    if (c.coef_mode != SS_COEF_FIXED && !(c.coef_ridge >= 0.f && c.coef_ridge < 3.0e38f))
        return fail(SS_ERR_INVALID_ARG, "coef_ridge must be finite and >= 0");
    if ((long long)c.batch * c.heads > (1ll << 31) / 2)
        return fail(SS_ERR_UNSUPPORTED, "batch * heads too large");
    ss_plan* pl = new (std::nothrow) ss_plan;
    if (pl == nullptr) return fail(SS_ERR_INVALID_ARG, "out of host memory");
    std::memset(pl, 0, sizeof *pl);
    pl->cfg = c;
    pl->cfg.ranks = nullptr;
    pl->cfg.dense_heads = nullptr;
    pl->off[0] = 0;
    pl->rmax = 0;
    for (int h = 0; h < c.heads; ++h) {
        const int r = c.ranks[h];
        if (r < 0 || r > c.dk) {
            delete pl;
            return fail(SS_ERR_INVALID_ARG, "ranks[%d] = %d outside 0..dk", h, r);
        }
        const bool dense = c.dense_heads != nullptr && c.dense_heads[h] != 0;
        if (dense) {
            if (r != c.dk) {
                delete pl;
                return fail(SS_ERR_INVALID_ARG, "dense head %d needs rank dk = %d (has %d)", h, c.dk, r);
            }
            pl->dense[h >> 5] |= 1u << (h & 31);
            pl->n_dense += 1;
            pl->ranks[h] = r;
            pl->off[h + 1] = pl->off[h] + r;
            continue;
        }
        if (c.coef_mode == SS_COEF_STATE && !ss::flush_map_fits(c.dk, c.dv, r)) {
            delete pl;
            return fail(SS_ERR_UNSUPPORTED, "ranks[%d] = %d: the state-dependent map needs rank <= dv and "
                        "room for U and its Gram matrix in the flush's tile buffer", h, r);
        }
        if (c.coef_mode == SS_COEF_LRD && !ss::flush_lrd_fits(c.dk, c.dv, r)) {
            delete pl;
            return fail(SS_ERR_UNSUPPORTED, "ranks[%d] = %d: the low-rank-plus-diagonal map needs room for "
                        "its pivots, diagonal and Gram matrix in the flush's tile buffer", h, r);
        }
        pl->ranks[h] = r;
        pl->off[h + 1] = pl->off[h] + r;
        if (r > pl->rmax) pl->rmax = r;
    }
    pl->R = pl->off[c.heads];
    pl->Wg = (c.window + 3) & ~3;
    // Every launch must fit one head (flush) or one warp (decode) in shared memory.
    const int rpad = (pl->rmax + 1 + 3) & ~3;
    const bool smap = c.coef_mode != SS_COEF_FIXED;
    const int fl = ss::flush_smem_bytes(c.family, c.dk, c.dv, c.window, rpad, smap);
    const int dec = ss::decode_smem_bytes(c.family, c.dk, c.dv, c.window - 1, pl->rmax, esize(pl), smap,
                                          pl->n_dense > 0);
    if (fl > kSmemLimit || dec > kSmemLimit) {
        const int rmax = pl->rmax;
        delete pl;
        return fail(SS_ERR_UNSUPPORTED, "window %d with max rank %d needs %d / %d bytes of shared memory",
                    c.window, rmax, fl, dec);
    }
    *out = pl;
    return ok();
}

ss_status ss_destroy(ss_plan* plan) {
    if (plan != nullptr) {
        if (plan->side) cudaStreamDestroy(plan->side);
        if (plan->fork) cudaEventDestroy(plan->fork);
        if (plan->join) cudaEventDestroy(plan->join);
    }
    delete plan;
    return ok();
}

ss_status ss_buffer_sizes(const ss_plan* pl, ss_sizes* out) {
    if (pl == nullptr || out == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or out is NULL");
    const ss_config& c = pl->cfg;
    const size_t BH = size_t(c.batch) * c.heads, K = c.dk, V = c.dv, W = c.window;
    std::memset(out, 0, sizeof *out);
    out->state = BH * K * V * 4;
    out->ring_k = BH * W * K * 2;
    out->ring_v = BH * W * V * 2;
    out->ring_gate = (c.family == SS_KDA ? BH * W * K : BH * pl->Wg) * 4;
    out->ring_beta = c.family == SS_MAMBA2 ? 0 : BH * pl->Wg * 4;
    out->sketch = size_t(c.batch) * pl->R * V * esize(pl);
    out->basis = size_t(pl->R) * K * 4;
    out->coef = size_t(pl->R) * K * 4;
    out->A = c.family == SS_MAMBA2 ? size_t(c.heads) * 4 : 0;
    out->q = BH * K * 2;
    out->k = BH * K * 2;
    out->v = BH * V * 2;
    out->gate = (c.family == SS_KDA ? BH * K : BH) * 4;
    out->beta = c.family == SS_MAMBA2 ? 0 : BH * 4;
    out->out = BH * V * 4;
    out->coef_state = state_map(pl) ? size_t(c.batch) * pl->R * K * esize(pl) : 0;
    out->total_rank = pl->R;
    out->gate_stride = c.family == SS_KDA ? c.window * c.dk : pl->Wg;
    return ok();
}

ss_status ss_get_phase(const ss_plan* pl, int32_t* phase, int32_t* sketch_valid) {
    if (pl == nullptr) return fail(SS_ERR_INVALID_ARG, "plan is NULL");
    if (phase) *phase = pl->phase;
    if (sketch_valid) *sketch_valid = pl->sketch_valid;
    return ok();
}

ss_status ss_set_phase(ss_plan* pl, int32_t phase, int32_t sketch_valid) {
    if (pl == nullptr) return fail(SS_ERR_INVALID_ARG, "plan is NULL");
    if (phase < 0 || phase > pl->cfg.window - 1)
        return fail(SS_ERR_INVALID_ARG, "phase %d outside 0..W-1", phase);
    pl->phase = phase;
    pl->sketch_valid = sketch_valid ? 1 : 0;
    return ok();
}

ss_status ss_prime(ss_plan* pl, const ss_buffers* b, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (pl->phase != 0)
        return fail(SS_ERR_SCHEDULE, "ss_prime needs phase 0 (phase is %d): flush first", pl->phase);
    REQUIRE_PTR(b->state, "bufs->state");
    REQUIRE_PTR(b->sketch, "bufs->sketch");
    REQUIRE_PTR(b->basis, "bufs->basis");
    CHECK(check_map(pl, b));
    CHECK(check_status(b));
    ss::FlushParams p = flush_params(pl, b, nullptr);
    p.n_ring = 0; p.has_token = 0; p.do_sketch = 1;
    p.stall = take_stall(pl);
    CHECK(launch_via(pl, "prime", [&] {
        return ss::launch_flush(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p, pl->rmax,
                                reinterpret_cast<cudaStream_t>(stream));
    }));
    CHECK(dense_copies(pl, p, reinterpret_cast<cudaStream_t>(stream)));
    pl->sketch_valid = 1;
    return ok();
}

ss_status ss_decode_step(ss_plan* pl, const ss_buffers* b, const ss_step_io* io, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (pl->phase > pl->cfg.window - 2)
        return fail(SS_ERR_SCHEDULE, "ss_decode_step at phase %d of window %d: the next step must flush",
                    pl->phase, pl->cfg.window);
    if (!pl->sketch_valid)
        return fail(SS_ERR_SCHEDULE, "ss_decode_step needs a current sketch (ss_prime or ss_flush first)");
    CHECK(check_ring(pl, b));
    REQUIRE_PTR(b->sketch, "bufs->sketch");
    if (state_map(pl)) CHECK(check_map(pl, b));
    else REQUIRE_PTR(b->coef, "bufs->coef");
    CHECK(check_io(pl, io));
    CHECK(check_status(b));
    ss::StepParams p = step_params(pl, b, io);
    p.stall = take_stall(pl);
    CHECK(launch_via(pl, "decode", [&] {
        return ss::launch_decode(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p, pl->rmax,
                                 reinterpret_cast<cudaStream_t>(stream));
    }));
    pl->phase += 1;
    return ok();
}

ss_status ss_flush(ss_plan* pl, const ss_buffers* b, const ss_step_io* io, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (io != nullptr && pl->phase != pl->cfg.window - 1)
        return fail(SS_ERR_SCHEDULE, "ss_flush with a token needs phase W-1 = %d (phase is %d)",
                    pl->cfg.window - 1, pl->phase);
    CHECK(check_ring(pl, b));
    if (io != nullptr) CHECK(check_io(pl, io));
    const bool sk = b->sketch != nullptr;
    if (sk) {
        REQUIRE_PTR(b->sketch, "bufs->sketch");
        REQUIRE_PTR(b->basis, "bufs->basis");
        CHECK(check_map(pl, b));
    }
    CHECK(check_status(b));
    ss::FlushParams p = flush_params(pl, b, io);
    p.n_ring = pl->phase;
    p.has_token = io != nullptr;
    p.do_sketch = sk;
    p.stall = take_stall(pl);
    CHECK(launch_via(pl, "flush", [&] {
        return ss::launch_flush(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p, pl->rmax,
                                reinterpret_cast<cudaStream_t>(stream));
    }));
    // The flush is queued: the window is applied whatever happens next.  If the
    // dense heads' copies fail to launch, the plan is left at phase 0 without a
    // valid sketch, so the next read asks for ss_prime instead of using it.
    pl->phase = 0;
    pl->sketch_valid = 0;
    CHECK(dense_copies(pl, p, reinterpret_cast<cudaStream_t>(stream)));
    pl->sketch_valid = sk;
    return ok();
}

ss_status ss_exact_step(ss_plan* pl, const ss_buffers* b, const ss_step_io* io, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (pl->phase != 0)
        return fail(SS_ERR_SCHEDULE, "ss_exact_step needs phase 0 (phase is %d)", pl->phase);
    REQUIRE_PTR(b->state, "bufs->state");
    if (pl->cfg.family == SS_MAMBA2) REQUIRE_PTR(b->A, "bufs->A");
    CHECK(check_io(pl, io));
    CHECK(check_status(b));
    ss::FlushParams p = flush_params(pl, b, io);
    p.n_ring = 0; p.has_token = 1; p.do_sketch = 0;
    p.stall = take_stall(pl);
    CHECK(launch_via(pl, "exact", [&] {
        return ss::launch_flush(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p, 0,
                                reinterpret_cast<cudaStream_t>(stream));
    }));
    pl->sketch_valid = 0;
    return ok();
}

ss_status ss_replay_step(ss_plan* pl, const ss_buffers* b, const ss_step_io* io, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (pl->phase > pl->cfg.window - 2)
        return fail(SS_ERR_SCHEDULE, "ss_replay_step at phase %d of window %d: the next step must flush",
                    pl->phase, pl->cfg.window);
    CHECK(check_ring(pl, b));
    CHECK(check_io(pl, io));
    CHECK(check_status(b));
    ss::StepParams p = step_params(pl, b, io);
    p.stall = take_stall(pl);
    CHECK(launch_via(pl, "replay", [&] {
        return ss::launch_replay(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p,
                                 reinterpret_cast<cudaStream_t>(stream));
    }));
    pl->phase += 1;
    return ok();
}

ss_status ss_step_mixed(ss_plan* pl, const ss_buffers* b, const ss_step_io* io, const int32_t* fill_in,
                        int32_t* fill_out, ss_stream stream) {
    if (pl == nullptr || b == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or bufs is NULL");
    if (pl->phase != 0)
        return fail(SS_ERR_SCHEDULE, "ss_step_mixed needs the plan at phase 0 (phase is %d)", pl->phase);
    if (!pl->sketch_valid)
        return fail(SS_ERR_SCHEDULE, "ss_step_mixed needs a current sketch (ss_prime first)");
    if (fill_in == nullptr || fill_out == nullptr) return fail(SS_ERR_INVALID_ARG, "fill_in or fill_out is NULL");
    if (reinterpret_cast<uintptr_t>(fill_in) % 4 || reinterpret_cast<uintptr_t>(fill_out) % 4)
        return fail(SS_ERR_ALIGNMENT, "fill_in and fill_out must be 4-byte aligned");
    if (static_cast<const void*>(fill_in) == static_cast<const void*>(fill_out))
        return fail(SS_ERR_INVALID_ARG, "fill_out must not alias fill_in");
    CHECK(check_ring(pl, b));
    REQUIRE_PTR(b->state, "bufs->state");
    REQUIRE_PTR(b->sketch, "bufs->sketch");
    REQUIRE_PTR(b->basis, "bufs->basis");
    if (state_map(pl)) CHECK(check_map(pl, b));
    else REQUIRE_PTR(b->coef, "bufs->coef");
    if (pl->cfg.family == SS_MAMBA2) REQUIRE_PTR(b->A, "bufs->A");
    CHECK(check_io(pl, io));
    CHECK(check_status(b));
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pl->side == nullptr) {                 // all three or none
        cudaStream_t side = nullptr;
        cudaEvent_t fork = nullptr, join = nullptr;
        cudaError_t e = cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (join) cudaEventDestroy(join);
            if (fork) cudaEventDestroy(fork);
            if (side) cudaStreamDestroy(side);
            return fail(SS_ERR_CUDA, "mixed step: side stream: %s", cudaGetErrorString(e));
        }
        pl->side = side;
        pl->fork = fork;
        pl->join = join;
    }
    const int stall = take_stall(pl);
    const int W = pl->cfg.window;
    // The flush (sequences at W-1) and the decode (the others) touch disjoint
    // sequences: the flush runs on the side stream, forked after the caller's
    // earlier work and joined back before anything the caller queues next, so
    // the two share the SMs (measured 6-12 % faster than one after the other;
    // capping the flush at 1-2 CTAs per SM to leave the decode room was slower).
    cudaError_t e = cudaEventRecord(pl->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->side, pl->fork, 0);
    if (e != cudaSuccess) return fail(SS_ERR_CUDA, "mixed step: fork: %s", cudaGetErrorString(e));
    // Once forked, the side stream is joined back whatever happens below, so a
    // failed launch never leaves a flush running unordered with the caller's
    // later work; the first failure is the status returned.
    ss_status s = SS_OK;
    {
        ss::FlushParams f = flush_params(pl, b, io);   // sequences with fill == W-1: the flush
        f.n_ring = W - 1;
        f.has_token = 1;
        f.do_sketch = 1;
        f.fill_in = fill_in;
        f.fill_out = fill_out;
        s = launch_via(pl, "mixed flush", [&] {
            return ss::launch_flush(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, f, pl->rmax, pl->side);
        });
        if (s == SS_OK) s = dense_copies(pl, f, pl->side);
    }
    if (s == SS_OK && W > 1) {                // sequences with fill < W-1: a non-flush step
        ss::StepParams p = step_params(pl, b, io);
        p.p = W - 2;                          // staging is sized for the longest window
        p.fill_in = fill_in;
        p.fill_out = fill_out;
        p.stall = stall;
        s = launch_via(pl, "mixed decode", [&] {
            return ss::launch_decode(pl->cfg.family, pl->cfg.dk, pl->cfg.dv, p, pl->rmax, st);
        });
    }
    e = cudaEventRecord(pl->join, pl->side);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, pl->join, 0);
    if (s != SS_OK) return s;
    if (e != cudaSuccess) return fail(SS_ERR_CUDA, "mixed step: join: %s", cudaGetErrorString(e));
    return ok();
}

ss_status ss_traffic_bytes(const ss_plan* pl, int32_t op, int32_t tau, ss_traffic* out) {
    if (pl == nullptr || out == nullptr) return fail(SS_ERR_INVALID_ARG, "plan or out is NULL");
    const ss_config& c = pl->cfg;
    const double K = c.dk, V = c.dv, W = c.window, B = c.batch, H = c.heads;
    const double sk = esize(pl);
    const bool m2 = c.family == SS_MAMBA2, kda = c.family == SS_KDA;
    const double gate = kda ? 4 * K : 4, beta = m2 ? 0 : 4;
    const double slot = 2 * K + 2 * V + gate + beta;
    const double tok = 2 * K + slot;          // q plus the slot's fields
    const double D = 4 * K * V;
    const double A = m2 ? 4 * H : 0;
    if (op == SS_OP_DECODE || op == SS_OP_REPLAY || op == SS_OP_FLUSH_NO_TOKEN) {
        if (tau < 0 || tau > c.window - 1) return fail(SS_ERR_INVALID_ARG, "tau %d outside 0..W-1", tau);
        if (op != SS_OP_FLUSH_NO_TOKEN && tau > c.window - 2)
            return fail(SS_ERR_INVALID_ARG, "tau %d: a non-flush step needs tau <= W-2", tau);
    }
    double R = pl->R;   // sum of ranks over heads
    double rd = 0, wr = 0, prd = 0, pwr = 0;
    const double bh = B * H;
    const double sketch_bytes = B * R * V * sk;          // U of every sequence
    const bool smap = c.coef_mode != SS_COEF_FIXED;
    // Dense-fallback heads: their dk sketch rows are the state copy; no
    // basis, coef or map rows of theirs are read, and each flush that
    // sketches reads their new state once more to write the copy.
    const double nd = pl->n_dense, Rs = R - nd * K;      // ranks of the sketched heads
    const double basis_s = Rs * K * 4;                   // basis / fixed map rows actually read
    const double copy_rd = B * nd * D;
    const double map_bytes = smap ? B * Rs * K * sk : 0; // per-sequence maps (state-dependent modes)
    const double paper_tg = B * Rs * (K + V) * 2 + (m2 ? 0 : B * Rs * W * 2) + B * nd * K * V * 2;
    switch (op) {
        case SS_OP_DECODE:
            rd = bh * (tok + tau * slot) + sketch_bytes + (smap ? map_bytes : basis_s) + A;
            wr = bh * (slot + 4 * V);
            prd = paper_tg;
            break;
        case SS_OP_FLUSH:
            rd = bh * (D + (W - 1) * slot + tok) + basis_s + copy_rd + A;
            wr = bh * (D + 4 * V) + sketch_bytes + map_bytes;
            prd = bh * D; pwr = bh * D;
            break;
        case SS_OP_FLUSH_NO_TOKEN:
            rd = bh * (D + tau * slot) + basis_s + copy_rd + A;
            wr = bh * D + sketch_bytes + map_bytes;
            prd = bh * D; pwr = bh * D;
            break;
        case SS_OP_PRIME:
            rd = bh * D + basis_s + copy_rd;
            wr = sketch_bytes + map_bytes;
            prd = bh * D;
            break;
        case SS_OP_EXACT:
            rd = bh * (D + tok) + A;
            wr = bh * (D + 4 * V);
            prd = bh * D; pwr = bh * D;
            break;
        case SS_OP_REPLAY:
            rd = bh * (D + tok + tau * slot) + A;
            wr = bh * (slot + 4 * V);
            prd = bh * D;
            break;
        case SS_OP_REPLAY_FLUSH:
            rd = bh * (D + (W - 1) * slot + tok) + A;
            wr = bh * (D + 4 * V);
            prd = bh * D; pwr = bh * D;
            break;
        default:
            return fail(SS_ERR_INVALID_ARG, "unknown op %d", op);
    }
    out->paper_read_bytes = prd;
    out->paper_write_bytes = pwr;
    out->read_bytes = rd;
    out->write_bytes = wr;
    return ok();
}

uint64_t ss_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

ss_status ss_debug_stall_next_copy(ss_plan* pl, int32_t stall) {
    if (pl == nullptr) return fail(SS_ERR_INVALID_ARG, "plan is NULL");
    pl->stall_next = stall ? 1 : 0;
    return ok();
}

ss_status ss_debug_fail_launch(ss_plan* pl, int32_t n) {
    if (pl == nullptr) return fail(SS_ERR_INVALID_ARG, "plan is NULL");
    if (n < 0) return fail(SS_ERR_INVALID_ARG, "n = %d < 0", n);
    pl->fail_launch = n;
    return ok();
}

const char* ss_status_string(ss_status s) {
    switch (s) {
        case SS_OK: return "SS_OK";
        case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG";
        case SS_ERR_ALIGNMENT: return "SS_ERR_ALIGNMENT";
        case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED";
        case SS_ERR_SCHEDULE: return "SS_ERR_SCHEDULE";
        case SS_ERR_CUDA: return "SS_ERR_CUDA";
    }
    return "unknown ss_status";
}

const char* ss_last_error_string(void) { return g_err.c_str(); }

}  // extern "C"
