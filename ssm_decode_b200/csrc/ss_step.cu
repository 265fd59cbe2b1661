// The ring-append + windowed-read kernels of the SketchSSM decode path.
//
//  * decode_kernel -- the non-flush step (project page, "Per step ·
//    Non-flush"; paper §3.2, §C.1): append the token at ring slot p, map the
//    query back through the buffered transitions (x_p = q,
//    x_{j-1} = M_j^T x_j, q~ = x_{-1}), collect the buffered updates' exact
//    term sum_j b_j (k_j . x_j) v_j, then read the sketch:
//    o^ = U (C q~) + that term.  The state is never touched.
//
//  * replay_kernel -- the ReplaySSM non-flush step: the same append and
//    sweep, then the exact read S0^T q~ + term over the full state.
//
// A (sequence, head) unit is served by one warp; lane l owns dk/32
// consecutive key channels and dv/32 consecutive value channels.  Everything
// a unit reads from HBM -- its live ring slots, its sketch rows and the
// step's token -- arrives by bulk asynchronous copies (cp.async.bulk) that
// complete on an mbarrier, issued by one lane, so a unit waits for memory
// once.  Every wait is bounded: when one runs out the kernel sets
// SS_DEVICE_TIMEOUT in the caller's status word and returns.
#include "ss_common.cuh"

namespace ss {
namespace {


// Per-unit shared-memory layout (byte offsets) of the staged window and token.
struct UnitSmem {
    int kraw, vraw, graw, gs, bs, ush, tq, tk, tv, tg, total;
};

__host__ __device__ inline UnitSmem unit_smem(int fam, int K, int V, int P, int ubytes) {
    UnitSmem L;
    int o = 0;
    const int P4 = (P + 3) & ~3;
    L.kraw = o; o += align16(P * K * 2);
    L.vraw = o; o += align16(P * V * 2);
    L.graw = o; o += align16(fam == KDA ? P * K * 4 : 0);
    L.gs = o;   o += align16(fam == KDA ? 0 : P4 * 4);
    L.bs = o;   o += align16(fam == MAMBA2 ? 0 : P4 * 4);
    L.ush = o;  o += align16(ubytes);
    L.tq = o;   o += align16(K * 2);
    L.tk = o;   o += align16(K * 2);
    L.tv = o;   o += align16(V * 2);
    L.tg = o;   o += align16(fam == KDA ? K * 4 : 0);
    L.total = o;
    return L;
}

// Bytes the bulk copies of one unit move: live ring slots 0..p-1, the sketch
// rows (decode only) and the step's token.
template <int FAM, int K, int V>
__device__ __forceinline__ unsigned unit_bytes(int P, int ubytes) {
    const int P4 = (P + 3) & ~3;
    unsigned n = P * K * 2 + P * V * 2 + K * 2 + K * 2 + V * 2 + ubytes;
    if (FAM == KDA) n += P * K * 4 + K * 4;
    else if (P > 0) n += P4 * 4;
    if (FAM != MAMBA2 && P > 0) n += P4 * 4;
    return n;
}

// Issue (one lane) the bulk copies of one unit: its live ring slots 0..P-1,
// `ubytes` of sketch rows from `usrc` (0 for replay) and the step's token.
template <int FAM, int K, int V>
__device__ __forceinline__ void stage_unit_bulk(const StepParams& p, long long unit, int P, unsigned char* sh,
                                                const UnitSmem& L, const void* usrc, int ubytes,
                                                uint64_t* bar, unsigned extra, const void* csrc = nullptr,
                                                int cbytes = 0) {
    mbar_expect_tx(bar, unit_bytes<FAM, K, V>(P, ubytes + cbytes) + extra);
    const long long ring_row = unit * p.W;
    if (P > 0) {
        const int P4 = (P + 3) & ~3;
        bulk_g2s(sh + L.kraw, p.ring_k + ring_row * K, P * K * 2, bar);
        bulk_g2s(sh + L.vraw, p.ring_v + ring_row * V, P * V * 2, bar);
        if (FAM == KDA) bulk_g2s(sh + L.graw, p.ring_gate + ring_row * K, P * K * 4, bar);
        else bulk_g2s(sh + L.gs, p.ring_gate + unit * p.Wg, P4 * 4, bar);
        if (FAM != MAMBA2) bulk_g2s(sh + L.bs, p.ring_beta + unit * p.Wg, P4 * 4, bar);
    }
    if (ubytes > 0) bulk_g2s(sh + L.ush, usrc, ubytes, bar);
    if (cbytes > 0) bulk_g2s(sh + L.ush + ubytes, csrc, cbytes, bar);     // the unit's own map rows
    bulk_g2s(sh + L.tq, p.tok_q + unit * K, K * 2, bar);
    bulk_g2s(sh + L.tk, p.tok_k + unit * K, K * 2, bar);
    bulk_g2s(sh + L.tv, p.tok_v + unit * V, V * 2, bar);
    if (FAM == KDA) bulk_g2s(sh + L.tg, p.tok_gate + unit * K, K * 4, bar);
}

// N consecutive bf16 values, widened.
template <int N>
__device__ __forceinline__ void ld_bf16(const uint16_t* src, float (&dst)[N]) {
    if constexpr (N == 8) {
        const uint4 w = *reinterpret_cast<const uint4*>(src);
        dst[0] = bf2f_lo(w.x); dst[1] = bf2f_hi(w.x); dst[2] = bf2f_lo(w.y); dst[3] = bf2f_hi(w.y);
        dst[4] = bf2f_lo(w.z); dst[5] = bf2f_hi(w.z); dst[6] = bf2f_lo(w.w); dst[7] = bf2f_hi(w.w);
    } else if constexpr (N == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(src);
        dst[0] = bf2f_lo(w.x); dst[1] = bf2f_hi(w.x); dst[2] = bf2f_lo(w.y); dst[3] = bf2f_hi(w.y);
    } else {
        static_assert(N == 2, "unsupported width");
        const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
        dst[0] = bf2f_lo(w); dst[1] = bf2f_hi(w);
    }
}

template <int N>
__device__ __forceinline__ void ld_f32(const float* src, float (&dst)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            const float4 f = reinterpret_cast<const float4*>(src)[i];
            dst[4 * i] = f.x; dst[4 * i + 1] = f.y; dst[4 * i + 2] = f.z; dst[4 * i + 3] = f.w;
        }
    } else {
        static_assert(N == 2, "unsupported width");
        const float2 f = *reinterpret_cast<const float2*>(src);
        dst[0] = f.x; dst[1] = f.y;
    }
}

template <int N>
__device__ __forceinline__ void st_f32(float* dst, const float (&v)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i)
            reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
        *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
    }
}

template <int N>
__device__ __forceinline__ void copy_bits(uint16_t* dst, const uint16_t* src) {
    if constexpr (N == 8) *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    else if constexpr (N == 4) *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
    else *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
}

// A unit is served by LPU lanes (16 or 32); lane l owns dk/LPU consecutive
// key channels and dv/LPU consecutive value channels.
template <int K, int V, int LPU>
struct Tok {
    static constexpr int EK = K / LPU, EV = V / LPU;
    float q[EK], k[EK], v[EV], g[EK];
    float gs, b;   // scalar decay input (Mamba-2 dt, GDN a) and update strength b
};

constexpr int lg2(int x) { return x <= 1 ? 0 : 1 + lg2(x / 2); }

// Sum over the LPU lanes of a unit (LPU-aligned lane groups).
template <int LPU>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int m = LPU / 2; m >= 1; m >>= 1) x += __shfl_xor_sync(FULL, x, m);
    return x;
}

// Reduce-scatter of NR per-lane partial sums over a unit's LPU lanes.
// Afterwards, with E = max(NR / LPU, 1), lane l holds in v[0 .. E) the totals
// of the entries owned by l: entry j lives in lane holder(j), slot(j).
template <int NR, int LPU>
struct Scatter {
    static constexpr int LH = lg2(NR) < lg2(LPU) ? lg2(NR) : lg2(LPU);   // halving levels
    static constexpr int E = NR >= LPU ? NR / LPU : 1;
    static constexpr int SH = lg2(LPU) - LH;                              // lanes per entry = 2^SH
    __device__ static int holder(int j) { return (j / E) << SH; }
    __device__ static int slot(int j) { return j % E; }
};

template <int NR, int LPU>
__device__ __forceinline__ void group_reduce_scatter(float (&v)[NR], int l) {
    using SC = Scatter<NR, LPU>;
#pragma unroll
    for (int lev = 0; lev < SC::LH; ++lev) {
        const int half = NR >> (lev + 1);
        const int m = (LPU / 2) >> lev;
        const bool upper = (l & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(FULL, send, m);
        }
    }
#pragma unroll
    for (int m = (1 << SC::SH) / 2; m >= 1; m >>= 1) v[0] += __shfl_xor_sync(FULL, v[0], m);
}

// Append the staged token, bit for bit, at ring slot p and widen it.
template <int FAM, int K, int V, int LPU>
__device__ __forceinline__ void append_token(const StepParams& p, long long unit, int l,
                                             const unsigned char* sh, const UnitSmem& L, float tgate,
                                             float tbeta, Tok<K, V, LPU>& tk) {
    constexpr int EK = K / LPU, EV = V / LPU;
    const uint16_t* tq = reinterpret_cast<const uint16_t*>(sh + L.tq) + l * EK;
    const uint16_t* tkk = reinterpret_cast<const uint16_t*>(sh + L.tk) + l * EK;
    const uint16_t* tv = reinterpret_cast<const uint16_t*>(sh + L.tv) + l * EV;
    const long long slot = unit * p.W + p.p;
    copy_bits<EK>(p.ring_k + slot * K + l * EK, tkk);
    copy_bits<EV>(p.ring_v + slot * V + l * EV, tv);
    ld_bf16<EK>(tq, tk.q);
    ld_bf16<EK>(tkk, tk.k);
    ld_bf16<EV>(tv, tk.v);
    if (FAM == KDA) {
        ld_f32<EK>(reinterpret_cast<const float*>(sh + L.tg) + l * EK, tk.g);
        st_f32<EK>(p.ring_gate + slot * K + l * EK, tk.g);
        tk.gs = 1.f;
    } else {
        tk.gs = tgate;
        if (l == 0) p.ring_gate[unit * p.Wg + p.p] = tk.gs;
#pragma unroll
        for (int e = 0; e < EK; ++e) tk.g[e] = 1.f;
    }
    if (FAM != MAMBA2) {
        tk.b = tbeta;
        if (l == 0) p.ring_beta[unit * p.Wg + p.p] = tk.b;
    } else {
        tk.b = tk.gs;   // b_j = dt_j
    }
}

// Mamba-2 window read in closed form (paper §C.1: q~ = d ⊙ q).  With no
// erase term, x_j = (prod_{i>j} a_i) q, so each buffered update's read is
// k_j . q scaled by a decay; the NR dot products are reduced together.
template <int NR, int K, int V, int LPU>
__device__ __forceinline__ void sweep_mamba2(const StepParams& p, int h, int l, int gbase,
                                             const unsigned char* sh, const UnitSmem& L,
                                             const Tok<K, V, LPU>& tk, float (&x)[K / LPU],
                                             float (&ob)[V / LPU]) {
    constexpr int EK = K / LPU, EV = V / LPU;
    using SC = Scatter<NR, LPU>;
    const int P = p.p;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw) + l * EK;
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw) + l * EV;
    const float* gs = reinterpret_cast<const float*>(sh + L.gs);
    float v[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        float acc = 0.f;
        if (j < P) {
            float kj[EK];
            ld_bf16<EK>(kraw + j * K, kj);
#pragma unroll
            for (int e = 0; e < EK; ++e) acc = fmaf(kj[e], tk.q[e], acc);
        } else if (j == P) {
#pragma unroll
            for (int e = 0; e < EK; ++e) acc = fmaf(tk.k[e], tk.q[e], acc);
        }
        v[j] = acc;
    }
    group_reduce_scatter<NR, LPU>(v, l);
    // decays: c_j = dt_j exp(A sum_{i>j} dt_i), computed for the entries this lane holds
    const float A = p.A[h];
    float pref = 0.f, my_pref[SC::E], my_dt[SC::E];
#pragma unroll
    for (int i = 0; i < SC::E; ++i) { my_pref[i] = 0.f; my_dt[i] = 0.f; }
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        const float dt = j < P ? gs[j] : (j == P ? tk.gs : 0.f);
        pref += dt;
        if (SC::holder(j) == (l & ~((1 << SC::SH) - 1))) { my_pref[SC::slot(j)] = pref; my_dt[SC::slot(j)] = dt; }
    }
    float c[SC::E];
#pragma unroll
    for (int i = 0; i < SC::E; ++i) c[i] = my_dt[i] * expf(A * (pref - my_pref[i])) * v[i];
    const float qs = expf(A * pref);
#pragma unroll
    for (int e = 0; e < EK; ++e) x[e] = qs * tk.q[e];
#pragma unroll
    for (int e = 0; e < EV; ++e) ob[e] = 0.f;
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        const float cj = __shfl_sync(FULL, c[SC::slot(j)], gbase + SC::holder(j));
        if (j < P) {
            float vj[EV];
            ld_bf16<EV>(vraw + j * V, vj);
#pragma unroll
            for (int e = 0; e < EV; ++e) ob[e] = fmaf(cj, vj[e], ob[e]);
        } else if (j == P) {
#pragma unroll
            for (int e = 0; e < EV; ++e) ob[e] = fmaf(cj, tk.v[e], ob[e]);
        }
    }
}

// Delta-rule (and generic) window read: the sequential backward sweep.
template <int FAM, int K, int V, int LPU>
__device__ __forceinline__ void sweep_seq(const StepParams& p, int h, int l, const unsigned char* sh,
                                          const UnitSmem& L, const Tok<K, V, LPU>& tk, float (&x)[K / LPU],
                                          float (&ob)[V / LPU]) {
    constexpr int EK = K / LPU, EV = V / LPU;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw) + l * EK;
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw) + l * EV;
    const float* graw = reinterpret_cast<const float*>(sh + L.graw) + l * EK;
    const float* gs = reinterpret_cast<const float*>(sh + L.gs);
    const float* bs = reinterpret_cast<const float*>(sh + L.bs);
    const float A = (FAM == MAMBA2) ? p.A[h] : 0.f;
#pragma unroll
    for (int e = 0; e < EK; ++e) x[e] = tk.q[e];
#pragma unroll
    for (int e = 0; e < EV; ++e) ob[e] = 0.f;
    for (int j = p.p; j >= 0; --j) {
        float kj[EK], vj[EV], aj[EK];
        float a_s, bj;
        if (j == p.p) {
#pragma unroll
            for (int e = 0; e < EK; ++e) { kj[e] = tk.k[e]; aj[e] = tk.g[e]; }
#pragma unroll
            for (int e = 0; e < EV; ++e) vj[e] = tk.v[e];
            a_s = tk.gs;
            bj = tk.b;
        } else {
            ld_bf16<EK>(kraw + j * K, kj);
            ld_bf16<EV>(vraw + j * V, vj);
            if (FAM == KDA) {
                ld_f32<EK>(graw + j * K, aj);
                a_s = 1.f;
            } else {
                a_s = gs[j];
            }
            bj = (FAM == MAMBA2) ? a_s : bs[j];
        }
        if (FAM == MAMBA2) a_s = expf(a_s * A);
        float k0 = 0.f, k1 = 0.f;
#pragma unroll
        for (int e = 0; e < EK; e += 2) { k0 = fmaf(kj[e], x[e], k0); k1 = fmaf(kj[e + 1], x[e + 1], k1); }
        const float bsx = bj * group_sum<LPU>(k0 + k1);
#pragma unroll
        for (int e = 0; e < EV; ++e) ob[e] = fmaf(bsx, vj[e], ob[e]);
#pragma unroll
        for (int e = 0; e < EK; ++e) {
            if (FAM == MAMBA2) x[e] *= a_s;
            else if (FAM == GDN) x[e] = a_s * fmaf(-bsx, kj[e], x[e]);
            else x[e] = aj[e] * fmaf(-bsx, kj[e], x[e]);
        }
    }
}

template <int FAM, int K, int V, int LPU>
__device__ __forceinline__ void window_read(const StepParams& p, int h, int l, int gbase, const unsigned char* sh,
                                            const UnitSmem& L, const Tok<K, V, LPU>& tk, float (&x)[K / LPU],
                                            float (&ob)[V / LPU]) {
    if constexpr (FAM == MAMBA2) {
        const int n = p.p + 1;
        if (n <= 8) sweep_mamba2<8, K, V, LPU>(p, h, l, gbase, sh, L, tk, x, ob);
        else if (n <= 16) sweep_mamba2<16, K, V, LPU>(p, h, l, gbase, sh, L, tk, x, ob);
        else sweep_mamba2<32, K, V, LPU>(p, h, l, gbase, sh, L, tk, x, ob);
    } else {
        sweep_seq<FAM, K, V, LPU>(p, h, l, sh, L, tk, x, ob);
    }
}

// ---------------------------------------------------------------------------
// decode_kernel.  A unit is served by a group of G = dec_gl(family) lanes,
// so a warp carries 32/G units (consecutive sequences of one head) through
// every instruction.  Each lane owns chunks of consecutive key and value
// channels (see Own), so a group's shared-memory reads are contiguous.  Dot
// products are reduced over the group with a butterfly.
//
// CTA (x, h) serves head h; one bulk copy stages the head's coefficient rows
// C (shared by the batch) once.  Warp w of CTA x takes the unit groups
// x*wpc + w + k*nb*wpc (k = 0, 1, ...) and runs them through NS staging
// buffers, issuing the bulk copies (live ring slots, sketch rows, token) of
// its next NS-1 groups before computing the current one.  The launcher
// below uses NS = 1 and one group per warp: on the bench shapes shared
// memory, not registers, bounds the units resident on an SM, and spending it
// on more CTAs measured faster than on deeper per-warp pipelines.
// ---------------------------------------------------------------------------
constexpr int DEC_WARPS = 4;              // warps per decode CTA
constexpr int DEC_UREG_ROWS = 16;         // sketch rows a unit can hold in registers

// Lanes per unit.  Mamba-2's reads are independent dot products, which 16
// lanes (2 units per warp) reduce cheaply; the delta rule's sweep is serial
// per unit, which 32 lanes (one unit per warp, more warps per SM) hide best.
__host__ __device__ constexpr int dec_gl(int fam) { return fam == MAMBA2 ? 16 : 32; }

// A unit's sketch (and own map) rows; with dense-fallback heads in the plan
// at least dk floats, which hold q~ for a dense head's read.
__host__ __device__ inline int dec_ubytes(int K, int V, int rmax, int esz, bool smap, bool dense_any) {
    const int ub = rmax * (V + (smap ? K : 0)) * esz;
    return dense_any && ub < K * 4 ? K * 4 : ub;
}

__host__ __device__ inline int dec_stage_bytes(int fam, int K, int V, int P, int ubytes) {
    return 16 + (32 / dec_gl(fam)) * unit_smem(fam, K, V, P, ubytes).total;   // mbarrier + the warp's units
}

// Sum over the G lanes of a unit.
template <int G>
__device__ __forceinline__ float gsum(float x) {
#pragma unroll
    for (int m = 1; m < G; m <<= 1) x += __shfl_xor_sync(FULL, x, m);
    return x;
}

// Channel ownership inside a unit's lane group, for a row of N values: lane
// l owns M chunks of CH consecutive channels, chunk m starting at
// m * G * CH + l * CH, so a group's 16-byte shared-memory reads of a bf16
// row cover contiguous bytes.
template <int N, int G>
struct Own {
    static constexpr int E = N / G;                  // channels per lane
    static constexpr int CH = E >= 8 ? 8 : E;         // channels per chunk
    static constexpr int M = E / CH;                  // chunks per lane
    __device__ static int base(int m, int l) { return m * G * CH + l * CH; }
};

__device__ __forceinline__ void unpack2(uint32_t w, float* d) { d[0] = bf2f_lo(w); d[1] = bf2f_hi(w); }

// This lane's channels of a row of N bf16 / fp32 values.
template <int N, int G>
__device__ __forceinline__ void row_bf16(const uint16_t* row, int l, float (&d)[N / G]) {
    using O = Own<N, G>;
#pragma unroll
    for (int m = 0; m < O::M; ++m) {
        const uint16_t* src = row + O::base(m, l);
        float* dd = d + m * O::CH;
        if constexpr (O::CH == 8) {
            const uint4 w = *reinterpret_cast<const uint4*>(src);
            unpack2(w.x, dd); unpack2(w.y, dd + 2); unpack2(w.z, dd + 4); unpack2(w.w, dd + 6);
        } else if constexpr (O::CH == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(src);
            unpack2(w.x, dd); unpack2(w.y, dd + 2);
        } else {
            static_assert(O::CH == 2, "chunk of 2, 4 or 8");
            unpack2(*reinterpret_cast<const uint32_t*>(src), dd);
        }
    }
}
template <int N, int G>
__device__ __forceinline__ void row_f32(const float* row, int l, float (&d)[N / G]) {
    using O = Own<N, G>;
#pragma unroll
    for (int m = 0; m < O::M; ++m) {
        if constexpr (O::CH == 2) {
            const float2 a = *reinterpret_cast<const float2*>(row + O::base(m, l));
            d[2 * m] = a.x; d[2 * m + 1] = a.y;
        } else {
#pragma unroll
            for (int q = 0; q < O::CH / 4; ++q) {
                const float4 a = *reinterpret_cast<const float4*>(row + O::base(m, l) + 4 * q);
                float* dd = d + m * O::CH + 4 * q;
                dd[0] = a.x; dd[1] = a.y; dd[2] = a.z; dd[3] = a.w;
            }
        }
    }
}
template <int N, int G, bool B16>
__device__ __forceinline__ void row_any(const void* row, int l, float (&d)[N / G]) {
    if constexpr (B16) row_bf16<N, G>(static_cast<const uint16_t*>(row), l, d);
    else row_f32<N, G>(static_cast<const float*>(row), l, d);
}
// Copy this lane's channels of a bf16 / fp32 row, bit for bit.
template <int N, int G>
__device__ __forceinline__ void copy_row_bf16(uint16_t* dst, const uint16_t* src, int l) {
    using O = Own<N, G>;
#pragma unroll
    for (int m = 0; m < O::M; ++m) {
        if constexpr (O::CH == 8)
            *reinterpret_cast<uint4*>(dst + O::base(m, l)) = *reinterpret_cast<const uint4*>(src + O::base(m, l));
        else if constexpr (O::CH == 4)
            *reinterpret_cast<uint2*>(dst + O::base(m, l)) = *reinterpret_cast<const uint2*>(src + O::base(m, l));
        else
            *reinterpret_cast<uint32_t*>(dst + O::base(m, l)) = *reinterpret_cast<const uint32_t*>(src + O::base(m, l));
    }
}
template <int N, int G>
__device__ __forceinline__ void copy_row_f32(float* dst, const float* src, int l) {
    using O = Own<N, G>;
#pragma unroll
    for (int m = 0; m < O::M; ++m) {
        if constexpr (O::CH == 2) {
            *reinterpret_cast<float2*>(dst + O::base(m, l)) = *reinterpret_cast<const float2*>(src + O::base(m, l));
        } else {
#pragma unroll
            for (int q = 0; q < O::CH / 4; ++q)
                reinterpret_cast<float4*>(dst + O::base(m, l))[q] = reinterpret_cast<const float4*>(src + O::base(m, l))[q];
        }
    }
}
template <int N, int G>
__device__ __forceinline__ void store_row_f32(float* dst, const float (&v)[N / G], int l) {
    using O = Own<N, G>;
#pragma unroll
    for (int m = 0; m < O::M; ++m) {
        if constexpr (O::CH == 2) {
            *reinterpret_cast<float2*>(dst + O::base(m, l)) = make_float2(v[2 * m], v[2 * m + 1]);
        } else {
#pragma unroll
            for (int q = 0; q < O::CH / 4; ++q) {
                const float* vv = v + m * O::CH + 4 * q;
                reinterpret_cast<float4*>(dst + O::base(m, l))[q] = make_float4(vv[0], vv[1], vv[2], vv[3]);
            }
        }
    }
}

template <int E>
__device__ __forceinline__ float dot(const float (&a)[E], const float (&b)[E]) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int e = 0; e < E; e += 2) { s0 = fmaf(a[e], b[e], s0); s1 = fmaf(a[e + 1], b[e + 1], s1); }
    return s0 + s1;
}
template <int E>
__device__ __forceinline__ void axpy(float a, const float (&x)[E], float (&y)[E]) {
#pragma unroll
    for (int e = 0; e < E; ++e) y[e] = fmaf(a, x[e], y[e]);
}

// UREG: the unit's sketch rows (bf16, at most DEC_UREG_ROWS, four channels a
// lane) are read straight into registers at the top of the unit instead of
// being staged in shared memory, which leaves room for more resident units.
template <int FAM, int K, int V, bool UB16, bool MIXED, bool UREG>
__global__ void __launch_bounds__(DEC_WARPS * 32) decode_kernel(const __grid_constant__ StepParams p,
                                                               int rmax, int ns, int stage_bytes) {
    constexpr int G = dec_gl(FAM), UPW = 32 / G;
    constexpr int EK = K / G, EV = V / G, ESZ = UB16 ? 2 : 4;
    static_assert(!UREG || (UB16 && EV == 4 && Own<V, G>::M == 1), "register sketch rows: bf16, 4 channels a lane");
    extern __shared__ __align__(16) unsigned char smem[];
    const int wpc = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane / G, l = lane % G;
    const int h = blockIdx.y;
    const int ngroups = (p.B + UPW - 1) / UPW;
    const int gstride = gridDim.x * wpc;
    const int g0 = blockIdx.x * wpc + warp;
    // A dense-fallback head (its sketch rows hold a copy of the state) stages
    // no sketch or map rows: its read streams the copy from HBM.
    const bool dense = head_dense(p.dense, h);
    const int off = p.off[h], r = dense ? 0 : p.off[h + 1] - off;
    const int P = p.p;
    // With the state-dependent map each unit stages its own C rows (r x dk,
    // sketch dtype) after its sketch rows; otherwise the CTA stages the
    // head's shared fp32 C once.
    const bool smap = p.cmap != nullptr;
    const UnitSmem L = unit_smem(FAM, K, V, P, UREG ? 0 : dec_ubytes(K, V, rmax, ESZ, smap, p.dense_any));
    const int cbytes = smap ? 0 : align16(rmax * K * 4);
    const float* csm = reinterpret_cast<const float*>(smem);
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + cbytes);
    unsigned char* wbase = smem + cbytes + 16 + warp * ns * stage_bytes;
    const bool stall = p.stall && blockIdx.x == 0 && blockIdx.y == 0 && warp == 0;

    auto bar = [&](int s) { return reinterpret_cast<uint64_t*>(wbase + s * stage_bytes); };
    unsigned pending = 0;      // bit s: stage s has copies in flight
    auto issue = [&](int it) {                             // this warp's group `it` into stage it % ns
        const int grp = g0 + it * gstride;
        if (grp >= ngroups) return;
        const int s = it % ns;
        if (l == 0) {
            const int b = grp * UPW + g;
            const int Pb = MIXED && b < p.B ? p.fill_in[b] : P;
            if (b < p.B && Pb >= 0 && Pb < p.W - 1)
                stage_unit_bulk<FAM, K, V>(p, (long long)b * p.H + h, Pb, wbase + s * stage_bytes + 16 + g * L.total, L,
                                           static_cast<const char*>(p.sketch) + (b * (long long)p.R + off) * (V * ESZ),
                                           UREG ? 0 : r * V * ESZ, bar(s), (stall && it == 0 && g == 0) ? 16u : 0u,
                                           smap ? static_cast<const char*>(p.cmap) + (b * (long long)p.R + off) * (K * ESZ)
                                                : nullptr,
                                           smap ? r * K * ESZ : 0);
            else
                mbar_arrive(bar(s));
        }
        pending |= 1u << s;
    };
    if (threadIdx.x == 0) mbar_init(cbar, 1);
    if (lane == 0 && g0 < ngroups)
        for (int s = 0; s < ns; ++s) mbar_init(bar(s), UPW);
    fence_mbar_init();
    __syncthreads();                                        // the only block barrier
    griddep_wait();                                         // the previous kernel's writes are visible
    griddep_launch_next();
    const float A = FAM == MAMBA2 ? p.A[h] : 0.f;
    if (threadIdx.x == 0) {
        mbar_expect_tx(cbar, smap ? 0 : r * K * 4);
        if (!smap && r > 0) bulk_g2s(smem, p.coef + (long long)off * K, r * K * 4, cbar);
    }
    if (g0 >= ngroups) return;                              // warp 0 always has a group
    for (int it = 0; it < ns; ++it) issue(it);              // before C arrives: the two latencies overlap
    bool ok = __all_sync(FULL, mbar_wait(cbar, 0));
    unsigned phases = 0;       // bit s: parity of the next phase of stage s
    int it = 0;
    for (int grp = g0; ok && grp < ngroups; ++it, grp += gstride) {
        const int s = it % ns;
        if (it > 0) issue(it + ns - 1);                        // its stage was freed by the last group
        const int b = grp * UPW + g;
        // this unit's ring position; in a mixed step, units at W-1 flush elsewhere
        const int Pu = MIXED ? (b < p.B ? p.fill_in[b] : 0) : P;
        const bool active = b < p.B && Pu >= 0 && Pu < p.W - 1;
        if (MIXED && b < p.B && (Pu < 0 || Pu > p.W - 1) && h == 0 && l == 0 && p.status)
            atomicOr(p.status, SS_DEVICE_BAD_FILL);              // neither decoded nor flushed
        const long long u = (long long)b * p.H + h;
        float tgate = 0.f, tbeta = 0.f;
        if (active) {
            if (FAM != KDA) tgate = p.tok_gate[u];
            if (FAM != MAMBA2) tbeta = p.tok_beta[u];
        }
        uint2 ureg[UREG ? DEC_UREG_ROWS : 1];                  // this lane's channels of the sketch rows
        if constexpr (UREG) {
            const uint16_t* urow = static_cast<const uint16_t*>(p.sketch) + (b * (long long)p.R + off) * V +
                                   Own<V, G>::base(0, l);
#pragma unroll
            for (int i = 0; i < DEC_UREG_ROWS; ++i)
                ureg[i] = active && i < r ? __ldg(reinterpret_cast<const uint2*>(urow + i * V)) : make_uint2(0u, 0u);
        }
        ok = __all_sync(FULL, mbar_wait(bar(s), (phases >> s) & 1u));
        if (!ok) break;
        phases ^= 1u << s;
        pending &= ~(1u << s);
        unsigned char* sh = wbase + s * stage_bytes + 16 + g * L.total;
        const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw);
        const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw);
        const float* graw = reinterpret_cast<const float*>(sh + L.graw);
        const float* gs = reinterpret_cast<const float*>(sh + L.gs);
        const float* bs = reinterpret_cast<const float*>(sh + L.bs);
        const uint16_t* tq = reinterpret_cast<const uint16_t*>(sh + L.tq);
        const uint16_t* tk = reinterpret_cast<const uint16_t*>(sh + L.tk);
        const uint16_t* tv = reinterpret_cast<const uint16_t*>(sh + L.tv);
        const float* tg = reinterpret_cast<const float*>(sh + L.tg);

        // 1. Append the token at ring slot Pu, bit for bit.
        if (active) {
            const long long slot = u * p.W + Pu;
            copy_row_bf16<K, G>(p.ring_k + slot * K, tk, l);
            copy_row_bf16<V, G>(p.ring_v + slot * V, tv, l);
            if (FAM == KDA) copy_row_f32<K, G>(p.ring_gate + slot * K, tg, l);
            else if (l == 0) p.ring_gate[u * p.Wg + Pu] = tgate;
            if (FAM != MAMBA2 && l == 0) p.ring_beta[u * p.Wg + Pu] = tbeta;
            if (MIXED && h == 0 && l == 0) p.fill_out[b] = Pu + 1;
        }

        // 2. Backward sweep from the token (j = P) to slot 0: x_P = q,
        //    x_{j-1} = M_j^T x_j, term += b_j (k_j . x_j) v_j.
        float x[EK], ob[EV], kj[EK], vj[EV];
        row_bf16<K, G>(tq, l, x);
        row_bf16<K, G>(tk, l, kj);
        row_bf16<V, G>(tv, l, vj);
#pragma unroll
        for (int e = 0; e < EV; ++e) ob[e] = 0.f;
        if constexpr (MIXED && FAM == MAMBA2) {
            // The uniform sweep below, 4 rows at a time, walked to the warp's
            // largest ring position: rows at or past this unit's own position
            // read as zero with unit decay (dt = 0).
            const int Pw = int(__reduce_max_sync(FULL, unsigned(active ? Pu : 0)));
            axpy<EV>(tgate * gsum<G>(dot<EK>(kj, x)), vj, ob);
            float gam = expf(A * tgate);
            int j = Pw - 1;
            for (; j >= 3; j -= 4) {
                float d[4], a[4], dt[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float kk[EK];
#pragma unroll
                    for (int e = 0; e < EK; ++e) kk[e] = 0.f;
                    dt[q] = 0.f;
                    if (j - q < Pu) {
                        row_bf16<K, G>(kraw + (j - q) * K, l, kk);
                        dt[q] = gs[j - q];
                    }
                    d[q] = dot<EK>(kk, x);
                    a[q] = expf(A * dt[q]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) d[q] = gsum<G>(d[q]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float vv[EV];
#pragma unroll
                    for (int e = 0; e < EV; ++e) vv[e] = 0.f;
                    if (j - q < Pu) row_bf16<V, G>(vraw + (j - q) * V, l, vv);
                    axpy<EV>(dt[q] * gam * d[q], vv, ob);
                    gam *= a[q];
                }
            }
            for (; j >= 0; --j) {
#pragma unroll
                for (int e = 0; e < EK; ++e) kj[e] = 0.f;
#pragma unroll
                for (int e = 0; e < EV; ++e) vj[e] = 0.f;
                float dt = 0.f;
                if (j < Pu) {
                    row_bf16<K, G>(kraw + j * K, l, kj);
                    row_bf16<V, G>(vraw + j * V, l, vj);
                    dt = gs[j];
                }
                const float dj = gsum<G>(dot<EK>(kj, x));
                axpy<EV>(dt * gam * dj, vj, ob);
                gam *= expf(A * dt);
            }
#pragma unroll
            for (int e = 0; e < EK; ++e) x[e] *= gam;
        } else if constexpr (MIXED) {
            // Units of one warp sit at different ring positions: every group
            // walks to the warp's largest position, rows past its own are
            // identities (zero key and value, unit decay).
            const int Pw = int(__reduce_max_sync(FULL, unsigned(active ? Pu : 0)));
            float gam = 1.f, aj[EK];
            {
                const float d = gsum<G>(dot<EK>(kj, x));
                if constexpr (FAM == MAMBA2) {
                    axpy<EV>(tgate * d, vj, ob);
                    gam = expf(A * tgate);
                } else {
                    const float t = tbeta * d;
                    axpy<EV>(t, vj, ob);
                    if constexpr (FAM == GDN) {
                        axpy<EK>(-t, kj, x);
                        gam = tgate;
                    } else {
                        row_f32<K, G>(tg, l, aj);
#pragma unroll
                        for (int e = 0; e < EK; ++e) x[e] = aj[e] * fmaf(-t, kj[e], x[e]);
                    }
                }
            }
            for (int j = Pw - 1; j >= 0; --j) {
                const bool own = j < Pu;
#pragma unroll
                for (int e = 0; e < EK; ++e) kj[e] = 0.f;
#pragma unroll
                for (int e = 0; e < EV; ++e) vj[e] = 0.f;
                float gj = FAM == MAMBA2 ? 0.f : 1.f, bj = 0.f;
                if (own) {
                    row_bf16<K, G>(kraw + j * K, l, kj);
                    row_bf16<V, G>(vraw + j * V, l, vj);
                    if (FAM != KDA) gj = gs[j];
                    if (FAM != MAMBA2) bj = bs[j];
                }
                const float d = gsum<G>(dot<EK>(kj, x));
                if constexpr (FAM == MAMBA2) {
                    axpy<EV>(gj * gam * d, vj, ob);            // gj = dt_j
                    gam *= expf(A * gj);
                } else if constexpr (FAM == GDN) {
                    const float t = bj * d;
                    axpy<EV>(gam * t, vj, ob);
                    axpy<EK>(-t, kj, x);
                    gam *= gj;
                } else {
#pragma unroll
                    for (int e = 0; e < EK; ++e) aj[e] = 1.f;
                    if (own) row_f32<K, G>(graw + j * K, l, aj);
                    const float t = bj * d;
                    axpy<EV>(t, vj, ob);
#pragma unroll
                    for (int e = 0; e < EK; ++e) x[e] = aj[e] * fmaf(-t, kj[e], x[e]);
                }
            }
            if constexpr (FAM != KDA) {
#pragma unroll
                for (int e = 0; e < EK; ++e) x[e] *= gam;
            }
        } else if constexpr (FAM == MAMBA2) {
            // No erase term: every read uses q, scaled by the later decays
            // (gam = prod_{i > j} a_i).  The rows are independent, so they
            // are taken 4 at a time: loads, dots and reductions overlap.
            axpy<EV>(tgate * gsum<G>(dot<EK>(kj, x)), vj, ob);
            float gam = expf(A * tgate);
            int j = P - 1;
            for (; j >= 3; j -= 4) {
                float d[4], a[4], dt[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float kk[EK];
                    row_bf16<K, G>(kraw + (j - q) * K, l, kk);
                    d[q] = dot<EK>(kk, x);
                    dt[q] = gs[j - q];
                    a[q] = expf(A * dt[q]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) d[q] = gsum<G>(d[q]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float vv[EV];
                    row_bf16<V, G>(vraw + (j - q) * V, l, vv);
                    axpy<EV>(dt[q] * gam * d[q], vv, ob);
                    gam *= a[q];
                }
            }
            for (; j >= 0; --j) {
                row_bf16<K, G>(kraw + j * K, l, kj);
                const float dj = gsum<G>(dot<EK>(kj, x));
                const float dt = gs[j];
                row_bf16<V, G>(vraw + j * V, l, vj);
                axpy<EV>(dt * gam * dj, vj, ob);
                gam *= expf(A * dt);
            }
#pragma unroll
            for (int e = 0; e < EK; ++e) x[e] *= gam;          // q~ = (prod a) q
        } else {
            // Delta rule: each row's read depends on the previous erase, so
            // the rows run in order; the next row is loaded while the current
            // one is reduced.
            float gam = 1.f;                                   // GDN: x_j = gam * y_j
            float aj[EK];
            {
                const float t = tbeta * gsum<G>(dot<EK>(kj, x));
                axpy<EV>(t, vj, ob);
                if constexpr (FAM == GDN) {
                    axpy<EK>(-t, kj, x);
                    gam = tgate;
                } else {
                    row_f32<K, G>(tg, l, aj);
#pragma unroll
                    for (int e = 0; e < EK; ++e) x[e] = aj[e] * fmaf(-t, kj[e], x[e]);
                }
            }
            if (P > 0) {
                row_bf16<K, G>(kraw + (P - 1) * K, l, kj);
                row_bf16<V, G>(vraw + (P - 1) * V, l, vj);
            }
            for (int j = P - 1; j >= 0; --j) {
                float kc[EK], vc[EV];
#pragma unroll
                for (int e = 0; e < EK; ++e) kc[e] = kj[e];
#pragma unroll
                for (int e = 0; e < EV; ++e) vc[e] = vj[e];
                const float bj = bs[j];
                if constexpr (FAM == KDA) row_f32<K, G>(graw + j * K, l, aj);
                const float part = dot<EK>(kc, x);
                if (j > 0) {
                    row_bf16<K, G>(kraw + (j - 1) * K, l, kj);
                    row_bf16<V, G>(vraw + (j - 1) * V, l, vj);
                }
                const float t = bj * gsum<G>(part);
                if constexpr (FAM == GDN) {
                    axpy<EV>(gam * t, vc, ob);
                    axpy<EK>(-t, kc, x);
                    gam *= gs[j];
                } else {
                    axpy<EV>(t, vc, ob);
#pragma unroll
                    for (int e = 0; e < EK; ++e) x[e] = aj[e] * fmaf(-t, kc[e], x[e]);
                }
            }
            if constexpr (FAM == GDN) {
#pragma unroll
                for (int e = 0; e < EK; ++e) x[e] *= gam;
            }
        }

        // 3. Coefficients c = C q~ and the sketched read o = U c + term,
        //    4 rows of C at a time.
        if (dense) {
            // Dense fallback: o += S0^T q~ from the state copy (row k = S0[k][:]);
            // q~ goes through the unit's buffer so every lane sees all of it.
            float* xs = reinterpret_cast<float*>(sh + L.ush);
            store_row_f32<K, G>(xs, x, l);
            __syncwarp();
            if (active) {
                const char* rows = static_cast<const char*>(p.sketch) + (b * (long long)p.R + off) * (V * ESZ);
                for (int k0 = 0; k0 < K; k0 += 8) {
                    float ui[8][EV];
#pragma unroll
                    for (int q = 0; q < 8; ++q) row_any<V, G, UB16>(rows + (k0 + q) * V * ESZ, l, ui[q]);
#pragma unroll
                    for (int q = 0; q < 8; ++q) axpy<EV>(xs[k0 + q], ui[q], ob);
                }
            }
        }
        const unsigned char* us = sh + L.ush;
        const unsigned char* cmu = us + r * V * ESZ;          // this unit's map rows (smap)
        auto crow = [&](int i, float (&ci)[EK]) {
            if (smap) row_any<K, G, UB16>(cmu + i * K * ESZ, l, ci);
            else row_f32<K, G>(csm + i * K, l, ci);
        };
        if constexpr (UREG) {
#pragma unroll
            for (int i0 = 0; i0 < DEC_UREG_ROWS; i0 += 4) {
                if (i0 < r) {
                    float c[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        c[q] = 0.f;
                        if (i0 + q < r) {
                            float ci[EK];
                            crow(i0 + q, ci);
                            c[q] = dot<EK>(ci, x);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) c[q] = gsum<G>(c[q]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {             // rows past r are zero
                        float ui[EV];
                        unpack2(ureg[i0 + q].x, ui);
                        unpack2(ureg[i0 + q].y, ui + 2);
                        axpy<EV>(c[q], ui, ob);
                    }
                }
            }
        }
        int i = UREG ? r : 0;
        for (; i + 4 <= r; i += 4) {
            float c[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float ci[EK];
                crow(i + q, ci);
                c[q] = dot<EK>(ci, x);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) c[q] = gsum<G>(c[q]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float ui[EV];
                row_any<V, G, UB16>(us + (i + q) * V * ESZ, l, ui);
                axpy<EV>(c[q], ui, ob);
            }
        }
        for (; i < r; ++i) {
            float ci[EK], ui[EV];
            crow(i, ci);
            const float c = gsum<G>(dot<EK>(ci, x));
            row_any<V, G, UB16>(us + i * V * ESZ, l, ui);
            axpy<EV>(c, ui, ob);
        }
        if (active) store_row_f32<V, G>(p.out + u * V, ob, l);
        __syncwarp();                                          // stage s is free again
    }
    if (!ok) {                                                 // a bounded wait ran out
        if (lane == 0) report_timeout(p.status);
        for (int t = 0; t < ns; ++t)                           // own copies: one more bounded wait
            if ((pending >> t) & 1u) mbar_wait(bar(t), (phases >> t) & 1u);
        if (warp == 0) mbar_wait(cbar, 0);
    }
}

// ---------------------------------------------------------------------------
// replay_kernel: exact windowed read S0^T q~ + term over the full state.  One
// warp per unit sweeps while the CTA holds the unit's state tile in registers.
// ---------------------------------------------------------------------------
template <int K>
__device__ __forceinline__ int kpad4(int c) {
    constexpr int R = K / 4;
    return (c / R) * (R + 4) + (c % R);
}

__host__ __device__ inline int replay_unit_bytes(int fam, int K, int V, int P) {
    return unit_smem(fam, K, V, P, 0).total + align16((K + 16) * 4) + align16(V * 4) + 16;   // + mbarrier
}

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
    const UnitSmem L = unit_smem(FAM, K, V, p.p, 0);
    unsigned char* sh = smem + hl * replay_unit_bytes(FAM, K, V, p.p);
    float* qt = reinterpret_cast<float*>(sh + L.total);
    float* obs = reinterpret_cast<float*>(sh + L.total + align16((K + 16) * 4));
    bool timed_out = false;

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
        uint64_t* bar = reinterpret_cast<uint64_t*>(sh + L.total + align16((K + 16) * 4) + align16(V * 4));
        if (lane == 0) {
            mbar_init(bar, 1);
            fence_mbar_init();
            stage_unit_bulk<FAM, K, V>(p, unit, p.p, sh, L, nullptr, 0, bar, p.stall && unit == 0 ? 16u : 0u);
        }
        const float tgate = FAM != KDA ? p.tok_gate[unit] : 0.f;
        const float tbeta = FAM != MAMBA2 ? p.tok_beta[unit] : 0.f;
        __syncwarp();
        timed_out = !mbar_wait(bar, 0);
        if (timed_out) {
            report_timeout(p.status);
            mbar_wait(bar, 0);
        } else {
            Tok<K, V, 32> tk;
            append_token<FAM, K, V, 32>(p, unit, lane, sh, L, tgate, tbeta, tk);
            float x[EK], ob[EV];
            window_read<FAM, K, V, 32>(p, h, lane, 0, sh, L, tk, x, ob);
#pragma unroll
            for (int e = 0; e < EK; ++e) qt[kpad4<K>(lane * EK + e)] = x[e];
#pragma unroll
            for (int e = 0; e < EV; ++e) obs[lane * EV + e] = ob[e];
        }
    }
    if (__syncthreads_or(timed_out)) return;
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
// One warp's staging buffer; with the state-dependent map (`smap`) each unit
// also stages its own map rows.
int decode_stage(int fam, int K, int V, int P, int rmax, int esz, bool smap, bool dense_any, bool ureg = false) {
    return dec_stage_bytes(fam, K, V, P, ureg ? 0 : dec_ubytes(K, V, rmax, esz, smap, dense_any));
}

// The CTA-wide part: the head's shared C (fixed map only) and its mbarrier.
int decode_cpart(int K, int rmax, bool smap) { return (smap ? 0 : align16(rmax * K * 4)) + 16; }

template <int FAM, int K, int V, bool UB16, bool MIXED, bool UREG>
cudaError_t decode_launch(const StepParams& p, int rmax, cudaStream_t stream) {
    constexpr int esz = UB16 ? 2 : 4, upw = 32 / dec_gl(FAM);
    const bool smap = p.cmap != nullptr;
    const int stage = decode_stage(FAM, K, V, p.p, rmax, esz, smap, p.dense_any != 0, UREG);
    const int cpart = decode_cpart(K, rmax, smap);
    if (cpart + stage > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    int wpc = DEC_WARPS;
    while (wpc > 1 && cpart + wpc * stage > SMEM_LIMIT) --wpc;
    const int bytes = cpart + wpc * stage;
    auto kern = decode_kernel<FAM, K, V, UB16, MIXED, UREG>;
    static KernelCache kc;
    cudaError_t e = ensure_smem(kern, kc, bytes);
    if (e != cudaSuccess) return e;
    const long long groups = (p.B + upw - 1) / upw;
    const long long nb = (groups + wpc - 1) / wpc;          // one group per warp
    return launch_pdl(kern, dim3(unsigned(nb), unsigned(p.H)), dim3(wpc * 32), bytes, stream, p, rmax, 1, stage);
}

// Resident CTAs per SM of a decode launch from its registers a thread and
// shared memory (1 KB of each SM's reserved per CTA).
int dec_blocks_per_sm(int regs, int bytes) {
    const int rr = (regs + 7) & ~7;
    const int by_regs = 65536 / (DEC_WARPS * 32 * rr);
    const int by_smem = SMEM_SM / (bytes + 1024);
    const int by_thr = 2048 / (DEC_WARPS * 32);
    return std::min(std::min(by_regs, by_smem), by_thr);
}

// Whether the register-held sketch rows fit more units on an SM than staging
// them: they free shared memory but cost registers.
template <int FAM, int K, int V, bool MIXED, bool OK>
bool dec_prefer_ureg(const StepParams& p, int rmax) {
    if constexpr (!OK) {
        return false;
    } else {
        constexpr int esz = 2;
        static KernelCache kc0, kc1;
        int r0 = 0, r1 = 0;
        if (cached_regs(decode_kernel<FAM, K, V, true, MIXED, false>, kc0, &r0) != cudaSuccess ||
            cached_regs(decode_kernel<FAM, K, V, true, MIXED, true>, kc1, &r1) != cudaSuccess)
            return false;
        const int cpart = decode_cpart(K, rmax, false);
        const int b0 = cpart + DEC_WARPS * decode_stage(FAM, K, V, p.p, rmax, esz, false, false, false);
        const int b1 = cpart + DEC_WARPS * decode_stage(FAM, K, V, p.p, rmax, esz, false, false, true);
        return dec_blocks_per_sm(r1, b1) > dec_blocks_per_sm(r0, b0);
    }
}

template <int FAM, int K, int V>
cudaError_t decode_t(const StepParams& p, int rmax, cudaStream_t stream) {
    // bf16 sketch rows of the fixed map, no dense-fallback head: held in
    // registers when that leaves more units resident
    constexpr int G = dec_gl(FAM);
    constexpr bool UREG_OK = V / G == 4 && Own<V, G>::M == 1;
    const bool ureg = UREG_OK && p.sketch_bf16 && p.cmap == nullptr && !p.dense_any && rmax <= DEC_UREG_ROWS &&
                      (p.fill_in ? dec_prefer_ureg<FAM, K, V, true, UREG_OK>(p, rmax)
                                  : dec_prefer_ureg<FAM, K, V, false, UREG_OK>(p, rmax));
    if (p.fill_in) {
        if (!p.sketch_bf16) return decode_launch<FAM, K, V, false, true, false>(p, rmax, stream);
        return ureg ? decode_launch<FAM, K, V, true, true, UREG_OK>(p, rmax, stream)
                    : decode_launch<FAM, K, V, true, true, false>(p, rmax, stream);
    }
    if (!p.sketch_bf16) return decode_launch<FAM, K, V, false, false, false>(p, rmax, stream);
    return ureg ? decode_launch<FAM, K, V, true, false, UREG_OK>(p, rmax, stream)
                : decode_launch<FAM, K, V, true, false, false>(p, rmax, stream);
}

template <int FAM, int K, int V>
cudaError_t replay_t(const StepParams& p, cudaStream_t stream) {
    const int per_head = replay_unit_bytes(FAM, K, V, p.p);
    int hpc = 128 / V;
    while (hpc > 1 && hpc * per_head > SMEM_LIMIT) --hpc;
    if (per_head > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    const long long units = (long long)p.B * p.H;
    const long long grid = (units + hpc - 1) / hpc;
    auto kern = replay_kernel<FAM, K, V>;
    static KernelCache kc;
    cudaError_t e = ensure_smem(kern, kc, hpc * per_head);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(grid)), dim3(hpc * V), hpc * per_head, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int family, int dk, int dv, const StepParams& p, int rmax, cudaStream_t stream) {
    SS_DISPATCH(decode_t, p, rmax, stream);
}

cudaError_t launch_replay(int family, int dk, int dv, const StepParams& p, cudaStream_t stream) {
    SS_DISPATCH(replay_t, p, stream);
}

int decode_smem_bytes(int family, int dk, int dv, int P, int rmax, int esz, bool smap, bool dense_any) {
    return decode_cpart(dk, rmax, smap) + decode_stage(family, dk, dv, P, rmax, esz, smap, dense_any);
}

}  // namespace ss
