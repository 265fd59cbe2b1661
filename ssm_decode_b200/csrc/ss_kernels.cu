// SketchSSM decode-path kernels for B200 (sm_100a).
//
// Three kernels cover every entry point of sketchssm.h:
//
//  * flush_kernel  -- streams each head's fp32 dk x dv state through
//    registers once: applies the buffered updates (ring slots, then the
//    step's own token), writes the state back, and, fused into the same pass,
//    the exact output S^T q and the sketch U = S^T Omega (paper §4.1 and
//    App. B as summarised on the paperlayer page: "sketch construction is
//    fused into the update kernel", project page "02 / How to Make a
//    Sketch").  It also serves ss_prime (zero updates), the ReplaySSM flush
//    (no sketch) and the Standard step (one update, no ring, no sketch).
//
//  * decode_kernel -- the non-flush step: appends the token to the ring and
//    forms o^ = U (C q~) + sum_j b_j (k_j . x_j) v_j from the staged ring
//    slots and the sketch, never touching the state (project page,
//    "Per step · Non-flush"; paper §3.2, §C.1).
//
//  * replay_kernel -- the ReplaySSM non-flush step: the same append and
//    backward sweep, then the exact read S0^T q~ over the full state.
//
// Thread layout of the state kernels: a head's state is split over V/4
// column groups x 4 row blocks; each thread keeps a (dk/4) x 4 tile in
// registers, loaded and stored with coalesced 16-byte accesses.  All
// reductions over dk are in-thread partial sums plus two butterfly
// shuffles across the four row blocks, which sit in the same warp.
//
// Scaled state: with scalar or per-channel decays the true state before
// update j is Diag(Gamma_j) S', where Gamma_j is the running product of the
// decays since the last renormalisation.  Folding Gamma into the keys
// (kw = Gamma ⊙ k for the delta rule's read, ku = k ⊘ Gamma for the write)
// turns every update into one FMA per state element for the write plus one
// for the delta rule's read, instead of a decay multiply on top.  When a
// running product leaves [2^-32, 2^32] the decay is folded into S' (one
// multiply per element) and the product restarts at 1, so nothing under- or
// overflows; a zero decay is applied exactly this way.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ss_internal.h"

namespace ss {
namespace {

constexpr int MAMBA2 = SS_MAMBA2, GDN = SS_GDN, KDA = SS_KDA;
constexpr unsigned FULL = 0xffffffffu;
constexpr float GAMMA_LO = 2.3283064365386963e-10f;  // 2^-32
constexpr float GAMMA_HI = 4294967296.0f;            // 2^32
constexpr int DEC_MAX_WARPS = 4;
constexpr int SMEM_LIMIT = 227 * 1024;

__device__ __forceinline__ float bf2f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }
__device__ __forceinline__ uint16_t f2bf(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Copy `bytes` (a multiple of 16) with `nthreads` cooperating threads.
__device__ __forceinline__ void stage(void* dst, const void* src, int bytes, int t, int nthreads) {
    for (int o = t * 16; o < bytes; o += nthreads * 16)
        cp_async16(static_cast<char*>(dst) + o, static_cast<const char*>(src) + o);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(FULL, x, m);
    return x;
}

__host__ __device__ __forceinline__ int align16(int x) { return (x + 15) & ~15; }

// ---------------------------------------------------------------------------
// flush_kernel
// ---------------------------------------------------------------------------
// Per-head shared-memory layout (byte offsets).  K-vectors used by the
// register tiles are stored "row-block padded": channel c lives at
// (c / R) * (R + 4) + c % R with R = dk/4, so the four row blocks of a warp
// hit disjoint banks.
struct FlushSmem {
    int kraw, vraw, graw, kw, ku, rn, pt, dco, meta, total;
};

__host__ __device__ inline FlushSmem flush_smem(int fam, int K, int V, int n, int rpad) {
    const int KP = K + 16, R = K / 4;
    FlushSmem L;
    int o = 0;
    L.kraw = o; o += align16(n * K * 2);
    L.vraw = o; o += align16(n * V * 2);
    L.graw = o; o += align16(fam == KDA ? n * K * 4 : 0);
    L.kw = o;   o += align16(fam == MAMBA2 ? 0 : n * KP * 4);
    L.ku = o;   o += align16(n * KP * 4);
    L.rn = o;   o += align16((n + 1) * KP * 4);
    L.pt = o;   o += align16(4 * (R * rpad + 4) * 4);
    L.dco = o;  o += align16(n * 4);
    L.meta = o; o += 16;
    L.total = o;
    return L;
}

template <int K>
__device__ __forceinline__ int kpad(int c) {
    constexpr int R = K / 4;
    return (c / R) * (R + 4) + (c % R);
}

template <int FAM, int K, int V>
__global__ void __launch_bounds__(128, 3) flush_kernel(const __grid_constant__ FlushParams p, int rpad) {
    constexpr int R = K / 4, KP = K + 16;
    extern __shared__ __align__(16) unsigned char smem[];

    const int hpc = blockDim.x / V;             // heads per CTA
    const int tid = threadIdx.x;
    const int hl = tid / V, t = tid % V;
    const int lane = tid & 31, cg = lane & 7, kq = lane >> 3;
    const int c0 = ((t >> 5) * 8 + cg) * 4;     // first of this thread's 4 columns
    const int row0 = kq * R;                    // first of this thread's R rows
    const long long unit = (long long)blockIdx.x * hpc + hl;   // flat (b, h)
    const bool active = unit < (long long)p.B * p.H;
    const int h = active ? int(unit % p.H) : 0;
    const long long b = active ? unit / p.H : 0;
    const int n = p.n_ring + p.has_token;

    const FlushSmem L = flush_smem(FAM, K, V, n, rpad);
    unsigned char* sh = smem + hl * L.total;
    uint16_t* kraw = reinterpret_cast<uint16_t*>(sh + L.kraw);
    uint16_t* vraw = reinterpret_cast<uint16_t*>(sh + L.vraw);
    float* graw = reinterpret_cast<float*>(sh + L.graw);
    float* kw = reinterpret_cast<float*>(sh + L.kw);
    float* ku = reinterpret_cast<float*>(sh + L.ku);
    float* rn = reinterpret_cast<float*>(sh + L.rn);
    float* pt = reinterpret_cast<float*>(sh + L.pt);
    float* dco = reinterpret_cast<float*>(sh + L.dco);
    int* meta = reinterpret_cast<int*>(sh + L.meta);

    // 1. The state tile goes straight to registers; all loads in flight at once.
    float* st = p.state + unit * (long long)(K * V);
    float s[R][4];
    if (active) {
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float4 x = __ldcs(reinterpret_cast<const float4*>(st + (row0 + i) * V + c0));
            s[i][0] = x.x; s[i][1] = x.y; s[i][2] = x.z; s[i][3] = x.w;
        }
    }

    const int r_h = (active && p.do_sketch) ? p.off[h + 1] - p.off[h] : 0;
    const int next = r_h + p.has_token;         // extended basis: [Omega_h | q]
    const int nch = (next + 3) / 4;

    // 2. Stage the window's keys, values (and KDA decays) with cp.async.
    if (active) {
        const long long ring_row = unit * p.W;
        stage(kraw, p.ring_k + ring_row * K, p.n_ring * K * 2, t, V);
        stage(vraw, p.ring_v + ring_row * V, p.n_ring * V * 2, t, V);
        if (FAM == KDA) stage(graw, p.ring_gate + ring_row * K, p.n_ring * K * 4, t, V);
        if (p.has_token) {
            stage(kraw + p.n_ring * K, p.tok_k + unit * K, K * 2, t, V);
            stage(vraw + p.n_ring * V, p.tok_v + unit * V, V * 2, t, V);
            if (FAM == KDA) stage(graw + p.n_ring * K, p.tok_gate + unit * K, K * 4, t, V);
        }
        cp_async_commit();
        // Extended basis, transposed into row-block-padded [dk][rpad] tiles.
        const int ecols = nch * 4;
        for (int idx = t; idx < K * ecols; idx += V) {
            const int e = idx / K, c = idx % K;
            float val = 0.f;
            if (e < r_h) val = __ldg(p.basis + (long long)(p.off[h] + e) * K + c);
            else if (e == r_h && p.has_token) val = bf2f(p.tok_q[unit * K + c]);
            pt[(c / R) * (R * rpad + 4) + (c % R) * rpad + e] = val;
        }
        cp_async_wait_all();
    }
    __syncthreads();

    // 3. One warp per head scans the decays: running products, renormalisation
    //    points, scaled keys kw / ku, and the per-update coefficient b_j.
    if (active && t < 32) {
        constexpr int CPL = K / 32;
        const long long gbase = unit * p.Wg;
        float gj = 1.f, bj = 0.f;               // lane j holds update j's (a_j, b_j)
        if (lane < n) {
            const bool tok = lane >= p.n_ring;
            if (FAM != KDA) gj = tok ? p.tok_gate[unit] : p.ring_gate[gbase + lane];
            if (FAM == MAMBA2) {
                bj = gj;                        // b_j = dt_j
                gj = expf(gj * p.A[h]);         // a_j = exp(dt_j A_h)
            } else {
                bj = tok ? p.tok_beta[unit] : p.ring_beta[gbase + lane];
            }
        }
        float gam[CPL];
#pragma unroll
        for (int m = 0; m < CPL; ++m) gam[m] = 1.f;
        unsigned mask = 0;
        int nrn = 0;
        for (int j = 0; j < n; ++j) {
            const float aj = __shfl_sync(FULL, gj, j);
            const float bjj = __shfl_sync(FULL, bj, j);
            float g[CPL];
            bool need = false;
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
                const int c = lane + 32 * m;
                g[m] = gam[m] * (FAM == KDA ? graw[j * K + c] : aj);
                need |= !(g[m] >= GAMMA_LO && g[m] <= GAMMA_HI);
            }
            if (__any_sync(FULL, need)) {       // fold the decay into S' before update j
#pragma unroll
                for (int m = 0; m < CPL; ++m) {
                    rn[nrn * KP + kpad<K>(lane + 32 * m)] = g[m];
                    gam[m] = 1.f;
                }
                mask |= 1u << j;
                ++nrn;
            } else {
#pragma unroll
                for (int m = 0; m < CPL; ++m) gam[m] = g[m];
            }
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
                const int c = lane + 32 * m;
                const float kv = bf2f(kraw[j * K + c]);
                if (FAM != MAMBA2) kw[j * KP + kpad<K>(c)] = gam[m] * kv;
                ku[j * KP + kpad<K>(c)] = kv * __frcp_rn(gam[m]);
            }
            if (lane == 0) dco[j] = bjj;
        }
#pragma unroll
        for (int m = 0; m < CPL; ++m) rn[nrn * KP + kpad<K>(lane + 32 * m)] = gam[m];
        if (lane == 0) { meta[0] = int(mask); meta[1] = nrn; }
    }
    __syncthreads();
    if (!active) return;

    // 4. Apply the updates: S' <- S' + ku_j d_j^T with d_j = b_j (v_j - S'^T kw_j).
    const unsigned mask = unsigned(meta[0]);
    const int blk = kq * (R + 4);
    int rni = 0;
    for (int j = 0; j < n; ++j) {
        if (mask & (1u << j)) {
            const float* g = rn + rni * KP + blk;
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 f = *reinterpret_cast<const float4*>(g + i);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    s[i][c] *= f.x; s[i + 1][c] *= f.y; s[i + 2][c] *= f.z; s[i + 3][c] *= f.w;
                }
            }
            ++rni;
        }
        float w[4] = {0.f, 0.f, 0.f, 0.f};
        if (FAM != MAMBA2) {
            const float* kr = kw + j * KP + blk;
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 f = *reinterpret_cast<const float4*>(kr + i);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    w[c] += f.x * s[i][c] + f.y * s[i + 1][c] + f.z * s[i + 2][c] + f.w * s[i + 3][c];
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                w[c] += __shfl_xor_sync(FULL, w[c], 8);
                w[c] += __shfl_xor_sync(FULL, w[c], 16);
            }
        }
        const float bjj = dco[j];
        const uint2 vv = *reinterpret_cast<const uint2*>(vraw + j * V + c0);
        float d[4];
        d[0] = bjj * (bf2f(vv.x & 0xffffu) - w[0]);
        d[1] = bjj * (bf2f(vv.x >> 16) - w[1]);
        d[2] = bjj * (bf2f(vv.y & 0xffffu) - w[2]);
        d[3] = bjj * (bf2f(vv.y >> 16) - w[3]);
        const float* kr = ku + j * KP + blk;
#pragma unroll
        for (int i = 0; i < R; i += 4) {
            const float4 f = *reinterpret_cast<const float4*>(kr + i);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                s[i][c] = fmaf(f.x, d[c], s[i][c]);
                s[i + 1][c] = fmaf(f.y, d[c], s[i + 1][c]);
                s[i + 2][c] = fmaf(f.z, d[c], s[i + 2][c]);
                s[i + 3][c] = fmaf(f.w, d[c], s[i + 3][c]);
            }
        }
    }
    {   // true state S = Diag(Gamma) S'
        const float* g = rn + meta[1] * KP + blk;
#pragma unroll
        for (int i = 0; i < R; i += 4) {
            const float4 f = *reinterpret_cast<const float4*>(g + i);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                s[i][c] *= f.x; s[i + 1][c] *= f.y; s[i + 2][c] *= f.z; s[i + 3][c] *= f.w;
            }
        }
    }

    // 5. Write the state back.
#pragma unroll
    for (int i = 0; i < R; ++i)
        __stcs(reinterpret_cast<float4*>(st + (row0 + i) * V + c0),
               make_float4(s[i][0], s[i][1], s[i][2], s[i][3]));

    // 6. Fused read-out against the extended basis [Omega_h | q], 4 columns of
    //    it per pass; the 4 row blocks reduce-scatter so that row block kq
    //    ends up with basis column 4*ch + kq.
    const int hi = kq >> 1, lo = kq & 1;
    for (int ch = 0; ch < nch; ++ch) {
        float acc[4][4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[e][c] = 0.f;
        const float* pp = pt + kq * (R * rpad + 4) + ch * 4;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float4 f = *reinterpret_cast<const float4*>(pp + i * rpad);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                acc[0][c] = fmaf(f.x, s[i][c], acc[0][c]);
                acc[1][c] = fmaf(f.y, s[i][c], acc[1][c]);
                acc[2][c] = fmaf(f.z, s[i][c], acc[2][c]);
                acc[3][c] = fmaf(f.w, s[i][c], acc[3][c]);
            }
        }
        float kept[2][4];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float mine = hi ? acc[2 + tt][c] : acc[tt][c];
                const float give = hi ? acc[tt][c] : acc[2 + tt][c];
                kept[tt][c] = mine + __shfl_xor_sync(FULL, give, 16);
            }
        float fin[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float mine = lo ? kept[1][c] : kept[0][c];
            const float give = lo ? kept[0][c] : kept[1][c];
            fin[c] = mine + __shfl_xor_sync(FULL, give, 8);
        }
        const int e = ch * 4 + kq;
        if (e < r_h) {
            const long long row = b * p.R + p.off[h] + e;
            if (p.sketch_bf16) {
                uint2 pk;
                pk.x = uint32_t(f2bf(fin[0])) | (uint32_t(f2bf(fin[1])) << 16);
                pk.y = uint32_t(f2bf(fin[2])) | (uint32_t(f2bf(fin[3])) << 16);
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.sketch) + row * V + c0) = pk;
            } else {
                *reinterpret_cast<float4*>(static_cast<float*>(p.sketch) + row * V + c0) =
                    make_float4(fin[0], fin[1], fin[2], fin[3]);
            }
        } else if (e == r_h && p.has_token) {
            *reinterpret_cast<float4*>(p.out + unit * V + c0) = make_float4(fin[0], fin[1], fin[2], fin[3]);
        }
    }
}

// ---------------------------------------------------------------------------
// ring append + backward sweep (shared by decode_kernel and replay_kernel)
// ---------------------------------------------------------------------------
struct StepSmem {
    int kraw, vraw, graw, gs, bs, ush, qt, ob, total;
};

__host__ __device__ inline StepSmem step_smem(int fam, int K, int V, int P, int ubytes, bool replay) {
    StepSmem L;
    int o = 0;
    const int P4 = (P + 3) & ~3;
    L.kraw = o; o += align16(P * K * 2);
    L.vraw = o; o += align16(P * V * 2);
    L.graw = o; o += align16(fam == KDA ? P * K * 4 : 0);
    L.gs = o;   o += align16(fam == KDA ? 0 : P4 * 4);
    L.bs = o;   o += align16(fam == MAMBA2 ? 0 : P4 * 4);
    L.ush = o;  o += align16(ubytes);
    L.qt = o;   o += align16(replay ? (K + 16) * 4 : 0);
    L.ob = o;   o += align16(replay ? V * 4 : 0);
    L.total = o;
    return L;
}

// Issue cp.async copies of ring slots 0..P-1 of one head (lane-cooperative).
template <int FAM, int K, int V>
__device__ __forceinline__ void stage_ring(const StepParams& p, long long unit, int lane,
                                           unsigned char* sh, const StepSmem& L) {
    const long long ring_row = unit * p.W;
    const int P = p.p;
    stage(sh + L.kraw, p.ring_k + ring_row * K, P * K * 2, lane, 32);
    stage(sh + L.vraw, p.ring_v + ring_row * V, P * V * 2, lane, 32);
    const int P4 = (P + 3) & ~3;
    if (FAM == KDA) stage(sh + L.graw, p.ring_gate + ring_row * K, P * K * 4, lane, 32);
    else stage(sh + L.gs, p.ring_gate + unit * p.Wg, P4 * 4, lane, 32);
    if (FAM != MAMBA2) stage(sh + L.bs, p.ring_beta + unit * p.Wg, P4 * 4, lane, 32);
}

template <int K, int V>
struct Token {
    static constexpr int EK = K / 32, EV = V / 32;
    float q[EK], k[EK], v[EV], g[EK];
    float gs, b;
};

template <int N>
__device__ __forceinline__ void load_bf16(const uint16_t* src, float (&dst)[N], uint32_t (&raw)[(N + 1) / 2]) {
    if constexpr (N == 4) {
        const uint2 x = *reinterpret_cast<const uint2*>(src);
        raw[0] = x.x; raw[1] = x.y;
    } else if constexpr (N == 2) {
        raw[0] = *reinterpret_cast<const uint32_t*>(src);
    }
#pragma unroll
    for (int e = 0; e < N; ++e) dst[e] = bf2f((raw[e / 2] >> (16 * (e & 1))) & 0xffffu);
}

template <int N>
__device__ __forceinline__ void store_raw(uint16_t* dst, const uint32_t (&raw)[(N + 1) / 2]) {
    if constexpr (N == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(raw[0], raw[1]);
    else *reinterpret_cast<uint32_t*>(dst) = raw[0];
}

// Read the step's token and append it, bit for bit, at ring slot p.
template <int FAM, int K, int V>
__device__ __forceinline__ void load_and_append(const StepParams& p, long long unit, int lane,
                                                Token<K, V>& tk) {
    constexpr int EK = K / 32, EV = V / 32;
    uint32_t rq[(EK + 1) / 2], rk[(EK + 1) / 2], rv[(EV + 1) / 2];
    load_bf16<EK>(p.tok_q + unit * K + lane * EK, tk.q, rq);
    load_bf16<EK>(p.tok_k + unit * K + lane * EK, tk.k, rk);
    load_bf16<EV>(p.tok_v + unit * V + lane * EV, tk.v, rv);
    const long long slot = unit * p.W + p.p;
    store_raw<EK>(p.ring_k + slot * K + lane * EK, rk);
    store_raw<EV>(p.ring_v + slot * V + lane * EV, rv);
    if (FAM == KDA) {
        const float* gsrc = p.tok_gate + unit * K + lane * EK;
        float* gdst = p.ring_gate + slot * K + lane * EK;
        if constexpr (EK == 4) {
            const float4 g4 = *reinterpret_cast<const float4*>(gsrc);
            *reinterpret_cast<float4*>(gdst) = g4;
            tk.g[0] = g4.x; tk.g[1] = g4.y; tk.g[2] = g4.z; tk.g[3] = g4.w;
        } else {
            const float2 g2 = *reinterpret_cast<const float2*>(gsrc);
            *reinterpret_cast<float2*>(gdst) = g2;
            tk.g[0] = g2.x; tk.g[1] = g2.y;
        }
        tk.gs = 1.f;
    } else {
        tk.gs = p.tok_gate[unit];
        if (lane == 0) p.ring_gate[unit * p.Wg + p.p] = tk.gs;
    }
    if (FAM != MAMBA2) {
        tk.b = p.tok_beta[unit];
        if (lane == 0) p.ring_beta[unit * p.Wg + p.p] = tk.b;
    } else {
        tk.b = tk.gs;   // b_j = dt_j
    }
}

// One backward-sweep update: ob += b (k . x) v; x <- M^T x.
template <int FAM, int EK, int EV>
__device__ __forceinline__ void sweep_one(float (&x)[EK], float (&ob)[EV], const float (&kj)[EK],
                                          const float (&vj)[EV], const float (&aj)[EK], float a_s,
                                          float bj) {
    float kx = 0.f;
#pragma unroll
    for (int e = 0; e < EK; ++e) kx = fmaf(kj[e], x[e], kx);
    kx = warp_sum(kx);
    const float bs = bj * kx;
#pragma unroll
    for (int e = 0; e < EV; ++e) ob[e] = fmaf(bs, vj[e], ob[e]);
#pragma unroll
    for (int e = 0; e < EK; ++e) {
        if (FAM == MAMBA2) x[e] *= a_s;
        else if (FAM == GDN) x[e] = a_s * fmaf(-bs, kj[e], x[e]);
        else x[e] = aj[e] * fmaf(-bs, kj[e], x[e]);
    }
}

// x <- q~ and ob <- buffered term, for the token plus staged slots p-1..0.
template <int FAM, int K, int V>
__device__ __forceinline__ void sweep(const StepParams& p, int h, int lane, const unsigned char* sh,
                                      const StepSmem& L, const Token<K, V>& tk, float (&x)[K / 32],
                                      float (&ob)[V / 32]) {
    constexpr int EK = K / 32, EV = V / 32;
    const float A = (FAM == MAMBA2) ? p.A[h] : 0.f;
#pragma unroll
    for (int e = 0; e < EK; ++e) x[e] = tk.q[e];
#pragma unroll
    for (int e = 0; e < EV; ++e) ob[e] = 0.f;
    {
        const float a_s = (FAM == MAMBA2) ? expf(tk.gs * A) : tk.gs;
        sweep_one<FAM, EK, EV>(x, ob, tk.k, tk.v, tk.g, a_s, tk.b);
    }
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw);
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw);
    const float* graw = reinterpret_cast<const float*>(sh + L.graw);
    const float* gs = reinterpret_cast<const float*>(sh + L.gs);
    const float* bs = reinterpret_cast<const float*>(sh + L.bs);
#pragma unroll 2
    for (int j = p.p - 1; j >= 0; --j) {
        float kj[EK], vj[EV], aj[EK];
        uint32_t rk[(EK + 1) / 2], rv[(EV + 1) / 2];
        load_bf16<EK>(kraw + j * K + lane * EK, kj, rk);
        load_bf16<EV>(vraw + j * V + lane * EV, vj, rv);
        float a_s = 1.f, bj;
        if (FAM == KDA) {
#pragma unroll
            for (int e = 0; e < EK; ++e) aj[e] = graw[j * K + lane * EK + e];
        } else {
            a_s = gs[j];
#pragma unroll
            for (int e = 0; e < EK; ++e) aj[e] = a_s;
        }
        if (FAM == MAMBA2) { bj = a_s; a_s = expf(a_s * A); }
        else bj = bs[j];
        sweep_one<FAM, EK, EV>(x, ob, kj, vj, aj, a_s, bj);
    }
}

// ---------------------------------------------------------------------------
// decode_kernel: one warp per (sequence, head)
// ---------------------------------------------------------------------------
template <int FAM, int K, int V>
__global__ void __launch_bounds__(DEC_MAX_WARPS * 32) decode_kernel(const __grid_constant__ StepParams p,
                                                                    int rmax) {
    constexpr int EK = K / 32, EV = V / 32;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
    if (unit >= (long long)p.B * p.H) return;   // whole warps only; no block barriers below
    const int h = int(unit % p.H);
    const long long b = unit / p.H;
    const int esz = p.sketch_bf16 ? 2 : 4;
    const StepSmem L = step_smem(FAM, K, V, p.p, rmax * V * esz, false);
    unsigned char* sh = smem + warp * L.total;
    const int off = p.off[h], r = p.off[h + 1] - off;

    stage_ring<FAM, K, V>(p, unit, lane, sh, L);
    stage(sh + L.ush, static_cast<const char*>(p.sketch) + (b * p.R + off) * (long long)(V * esz),
          r * V * esz, lane, 32);
    cp_async_commit();

    Token<K, V> tk;
    load_and_append<FAM, K, V>(p, unit, lane, tk);
    cp_async_wait_all();
    __syncwarp();

    float x[EK], ob[EV];
    sweep<FAM, K, V>(p, h, lane, sh, L, tk, x, ob);

    // c_i = C_i . q~ ; o^ = sum_i c_i u_i + ob
    float o[EV];
#pragma unroll
    for (int e = 0; e < EV; ++e) o[e] = ob[e];
    const float* crow = p.coef + (long long)off * K + lane * EK;
    for (int i = 0; i < r; ++i) {
        float part = 0.f;
        if constexpr (EK == 4) {
            const float4 c4 = __ldg(reinterpret_cast<const float4*>(crow + i * K));
            part = c4.x * x[0] + c4.y * x[1] + c4.z * x[2] + c4.w * x[3];
        } else {
            const float2 c2 = __ldg(reinterpret_cast<const float2*>(crow + i * K));
            part = c2.x * x[0] + c2.y * x[1];
        }
        const float ci = warp_sum(part);
        if (p.sketch_bf16) {
            const uint16_t* u = reinterpret_cast<const uint16_t*>(sh + L.ush) + i * V + lane * EV;
            float uf[EV];
            uint32_t ru[(EV + 1) / 2];
            load_bf16<EV>(u, uf, ru);
#pragma unroll
            for (int e = 0; e < EV; ++e) o[e] = fmaf(ci, uf[e], o[e]);
        } else {
            const float* u = reinterpret_cast<const float*>(sh + L.ush) + i * V + lane * EV;
#pragma unroll
            for (int e = 0; e < EV; ++e) o[e] = fmaf(ci, u[e], o[e]);
        }
    }
    float* dst = p.out + unit * V + lane * EV;
    if constexpr (EV == 4) *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    else *reinterpret_cast<float2*>(dst) = make_float2(o[0], o[1]);
}

// ---------------------------------------------------------------------------
// replay_kernel: exact windowed read S0^T q~ + ob over the full state
// ---------------------------------------------------------------------------
template <int FAM, int K, int V>
__global__ void __launch_bounds__(128) replay_kernel(const __grid_constant__ StepParams p) {
    constexpr int R = K / 4, EK = K / 32, EV = V / 32;
    extern __shared__ __align__(16) unsigned char smem[];
    const int hpc = blockDim.x / V;
    const int tid = threadIdx.x, hl = tid / V, t = tid % V;
    const int lane = tid & 31, cg = lane & 7, kq = lane >> 3;
    const int c0 = ((t >> 5) * 8 + cg) * 4, row0 = kq * R;
    const long long unit = (long long)blockIdx.x * hpc + hl;
    const bool active = unit < (long long)p.B * p.H;
    const int h = active ? int(unit % p.H) : 0;
    const StepSmem L = step_smem(FAM, K, V, p.p, 0, true);
    unsigned char* sh = smem + hl * L.total;
    float* qt = reinterpret_cast<float*>(sh + L.qt);
    float* obs = reinterpret_cast<float*>(sh + L.ob);

    const float* st = p.state + unit * (long long)(K * V);
    float s[R][4];
    if (active) {
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float4 x = __ldcs(reinterpret_cast<const float4*>(st + (row0 + i) * V + c0));
            s[i][0] = x.x; s[i][1] = x.y; s[i][2] = x.z; s[i][3] = x.w;
        }
    }
    if (active && t < 32) {
        stage_ring<FAM, K, V>(p, unit, lane, sh, L);
        cp_async_commit();
        Token<K, V> tk;
        load_and_append<FAM, K, V>(p, unit, lane, tk);
        cp_async_wait_all();
        __syncwarp();
        float x[EK], ob[EV];
        sweep<FAM, K, V>(p, h, lane, sh, L, tk, x, ob);
#pragma unroll
        for (int e = 0; e < EK; ++e) qt[kpad<K>(lane * EK + e)] = x[e];
#pragma unroll
        for (int e = 0; e < EV; ++e) obs[lane * EV + e] = ob[e];
    }
    __syncthreads();
    if (!active) return;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* qr = qt + kq * (R + 4);
#pragma unroll
    for (int i = 0; i < R; i += 4) {
        const float4 f = *reinterpret_cast<const float4*>(qr + i);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            acc[c] += f.x * s[i][c] + f.y * s[i + 1][c] + f.z * s[i + 2][c] + f.w * s[i + 3][c];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        acc[c] += __shfl_xor_sync(FULL, acc[c], 8);
        acc[c] += __shfl_xor_sync(FULL, acc[c], 16);
    }
    if (kq == 0) {
        const float4 o4 = *reinterpret_cast<const float4*>(obs + c0);
        *reinterpret_cast<float4*>(p.out + unit * V + c0) =
            make_float4(acc[0] + o4.x, acc[1] + o4.y, acc[2] + o4.z, acc[3] + o4.w);
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename Kern>
cudaError_t set_smem(Kern kern, int bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int FAM, int K, int V>
cudaError_t flush_t(const FlushParams& p, int rmax, cudaStream_t stream) {
    const int n = p.n_ring + p.has_token;
    const int rpad = ((p.do_sketch ? rmax : 0) + p.has_token + 3) & ~3;
    const int per_head = flush_smem(FAM, K, V, n, rpad).total;
    int hpc = 128 / V;
    while (hpc > 1 && hpc * per_head > SMEM_LIMIT) --hpc;
    if (per_head > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    const long long units = (long long)p.B * p.H;
    const long long grid = (units + hpc - 1) / hpc;
    auto kern = flush_kernel<FAM, K, V>;
    cudaError_t e = set_smem(kern, hpc * per_head);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(grid)), dim3(hpc * V), hpc * per_head, stream>>>(p, rpad);
    return cudaGetLastError();
}

template <int FAM, int K, int V>
cudaError_t decode_t(const StepParams& p, int rmax, cudaStream_t stream) {
    const int esz = p.sketch_bf16 ? 2 : 4;
    const int per_warp = step_smem(FAM, K, V, p.p, rmax * V * esz, false).total;
    if (per_warp > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    int wpc = DEC_MAX_WARPS;
    while (wpc > 1 && wpc * per_warp > SMEM_LIMIT) --wpc;
    const long long units = (long long)p.B * p.H;
    const long long grid = (units + wpc - 1) / wpc;
    auto kern = decode_kernel<FAM, K, V>;
    cudaError_t e = set_smem(kern, wpc * per_warp);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(grid)), dim3(wpc * 32), wpc * per_warp, stream>>>(p, rmax);
    return cudaGetLastError();
}

template <int FAM, int K, int V>
cudaError_t replay_t(const StepParams& p, cudaStream_t stream) {
    const int per_head = step_smem(FAM, K, V, p.p, 0, true).total;
    int hpc = 128 / V;
    while (hpc > 1 && hpc * per_head > SMEM_LIMIT) --hpc;
    if (per_head > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    const long long units = (long long)p.B * p.H;
    const long long grid = (units + hpc - 1) / hpc;
    auto kern = replay_kernel<FAM, K, V>;
    cudaError_t e = set_smem(kern, hpc * per_head);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(grid)), dim3(hpc * V), hpc * per_head, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

#define SS_DISPATCH(FN, ...)                                                              \
    do {                                                                                  \
        const int key = family * 100 + (dk == 128 ? 10 : 0) + (dv == 128 ? 1 : 0);          \
        switch (key) {                                                                    \
            case 0: return FN<MAMBA2, 64, 64>(__VA_ARGS__);                               \
            case 1: return FN<MAMBA2, 64, 128>(__VA_ARGS__);                              \
            case 10: return FN<MAMBA2, 128, 64>(__VA_ARGS__);                             \
            case 11: return FN<MAMBA2, 128, 128>(__VA_ARGS__);                            \
            case 100: return FN<GDN, 64, 64>(__VA_ARGS__);                                \
            case 101: return FN<GDN, 64, 128>(__VA_ARGS__);                               \
            case 110: return FN<GDN, 128, 64>(__VA_ARGS__);                               \
            case 111: return FN<GDN, 128, 128>(__VA_ARGS__);                              \
            case 200: return FN<KDA, 64, 64>(__VA_ARGS__);                                \
            case 201: return FN<KDA, 64, 128>(__VA_ARGS__);                               \
            case 210: return FN<KDA, 128, 64>(__VA_ARGS__);                               \
            case 211: return FN<KDA, 128, 128>(__VA_ARGS__);                              \
            default: return cudaErrorInvalidValue;                                        \
        }                                                                                 \
    } while (0)

cudaError_t launch_flush(int family, int dk, int dv, const FlushParams& p, int rmax, cudaStream_t stream) {
    SS_DISPATCH(flush_t, p, rmax, stream);
}

cudaError_t launch_decode(int family, int dk, int dv, const StepParams& p, int rmax, cudaStream_t stream) {
    SS_DISPATCH(decode_t, p, rmax, stream);
}

cudaError_t launch_replay(int family, int dk, int dv, const StepParams& p, cudaStream_t stream) {
    SS_DISPATCH(replay_t, p, stream);
}

int flush_smem_bytes(int family, int dk, int dv, int n, int rpad) {
    return flush_smem(family, dk, dv, n, rpad).total;
}

int step_smem_bytes(int family, int dk, int dv, int P, int ubytes, bool replay) {
    return step_smem(family, dk, dv, P, ubytes, replay).total;
}

}  // namespace ss
