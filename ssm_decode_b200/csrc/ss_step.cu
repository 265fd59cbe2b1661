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
// A (sequence, head) unit is served by a group of lanes (16 in decode_kernel,
// 32 in replay_kernel); lane l owns a slice of consecutive key channels and
// value channels.  Everything a unit reads -- its live ring slots, its sketch
// rows and the step's token -- is requested with cp.async at kernel entry, so
// a unit waits for memory once.  The units of a decode CTA share one head, so
// the head's coefficient map C is staged once per CTA.
#include "ss_common.cuh"

namespace ss {
namespace {

#ifndef SS_DEC_MAX_WARPS
#define SS_DEC_MAX_WARPS 4
#endif
constexpr int DEC_MAX_WARPS = SS_DEC_MAX_WARPS;   // warps (= units) per decode CTA

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

// Issue (one lane) the bulk copies of one unit: its live ring slots 0..p-1,
// `ubytes` of sketch rows from `usrc` (0 for replay) and the step's token.
template <int FAM, int K, int V>
__device__ __forceinline__ void stage_unit_bulk(const StepParams& p, long long unit, unsigned char* sh,
                                                const UnitSmem& L, const void* usrc, int ubytes,
                                                uint64_t* bar, unsigned extra) {
    const int P = p.p;
    mbar_expect_tx(bar, unit_bytes<FAM, K, V>(P, ubytes) + extra);
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

// c = C q~ for nr <= NR rows of C (shared memory), reduce-scattered; then
// o += sum_i c_i u_i, the sketch rows read through `U(i, u)`.
template <int NR, int K, int V, int LPU, typename LoadU>
__device__ __forceinline__ void readout(const float* csm, int nr, int l, int gbase, const float (&x)[K / LPU],
                                        float (&o)[V / LPU], LoadU U) {
    constexpr int EK = K / LPU, EV = V / LPU;
    using SC = Scatter<NR, LPU>;
    float v[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        float acc = 0.f;
        if (i < nr) {
            float cr[EK];
            ld_f32<EK>(csm + i * K + l * EK, cr);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int e = 0; e < EK; e += 2) { a0 = fmaf(cr[e], x[e], a0); a1 = fmaf(cr[e + 1], x[e + 1], a1); }
            acc = a0 + a1;
        }
        v[i] = acc;
    }
    group_reduce_scatter<NR, LPU>(v, l);
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const float ci = __shfl_sync(FULL, v[SC::slot(i)], gbase + SC::holder(i));
        if (i < nr) {
            float u[EV];
            U(i, u);
#pragma unroll
            for (int e = 0; e < EV; ++e) o[e] = fmaf(ci, u[e], o[e]);
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
// decode_kernel: DEC_LPU lanes per unit.  CTA (x, h) serves head h for
// consecutive sequences: one bulk copy stages h's coefficient map C, and the
// first lane of each unit issues that unit's bulk copies; everything lands on
// mbarriers, so each unit waits for memory once.
// ---------------------------------------------------------------------------
#ifndef SS_DEC_LPU
#define SS_DEC_LPU 16
#endif
constexpr int DEC_LPU = SS_DEC_LPU;

__host__ __device__ inline int dec_unit_bytes(int fam, int K, int V, int P, int ubytes) {
    return 16 + unit_smem(fam, K, V, P, ubytes).total;      // mbarrier + staged unit
}

template <int FAM, int K, int V>
__global__ void __launch_bounds__(DEC_MAX_WARPS * 32) decode_kernel(const __grid_constant__ StepParams p,
                                                                    int rmax) {
    constexpr int LPU = DEC_LPU, UPW = 32 / LPU, EK = K / LPU, EV = V / LPU;
    extern __shared__ __align__(16) unsigned char smem[];
    const int wpc = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hw = lane / LPU, l = lane % LPU, gbase = hw * LPU;
    const int h = blockIdx.y;
    const int b = (blockIdx.x * wpc + warp) * UPW + hw;
    const bool active = b < p.B;
    const long long unit = (long long)b * p.H + h;
    const int esz = p.sketch_bf16 ? 2 : 4;
    const int off = p.off[h], r = p.off[h + 1] - off;
    const int ubytes = r * V * esz;
    const UnitSmem L = unit_smem(FAM, K, V, p.p, rmax * V * esz);
    const int cbytes = align16(rmax * K * 4);
    const float* csm = reinterpret_cast<const float*>(smem);
    uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + cbytes);
    unsigned char* ubase = smem + cbytes + 16 + (warp * UPW + hw) * dec_unit_bytes(FAM, K, V, p.p, rmax * V * esz);
    uint64_t* ubar = reinterpret_cast<uint64_t*>(ubase);
    unsigned char* sh = ubase + 16;

    if (threadIdx.x == 0) mbar_init(cbar, 1);
    if (l == 0) mbar_init(ubar, 1);
    fence_mbar_init();
    __syncthreads();                                        // the only block barrier
    const bool stall = p.stall && blockIdx.x == 0 && blockIdx.y == 0;
    if (threadIdx.x == 0) {
        mbar_expect_tx(cbar, r * K * 4 + (stall ? 16u : 0u));
        if (r > 0) bulk_g2s(smem, p.coef + (long long)off * K, r * K * 4, cbar);
    }
    if (active && l == 0)
        stage_unit_bulk<FAM, K, V>(p, unit, sh, L,
                                   static_cast<const char*>(p.sketch) + (b * (long long)p.R + off) * (V * esz),
                                   ubytes, ubar, 0u);
    float tgate = 0.f, tbeta = 0.f;                         // token scalars: plain loads
    if (active) {
        if (FAM != KDA) tgate = p.tok_gate[unit];
        if (FAM != MAMBA2) tbeta = p.tok_beta[unit];
    }
    bool ok = mbar_wait(cbar, 0);
    if (active) ok = mbar_wait(ubar, 0) && ok;
    if (!ok) {                                              // a bounded wait ran out
        report_timeout(p.status);
        mbar_wait(cbar, 0);                                 // give own copies one more bounded wait
        if (active) mbar_wait(ubar, 0);
        return;
    }
    if (__all_sync(FULL, !active)) return;

    // Lanes whose unit lies past the batch take part in the shuffles (on
    // zeros, inside their own lane group) but store nothing.
    Tok<K, V, LPU> tk;
    if (active) {
        append_token<FAM, K, V, LPU>(p, unit, l, sh, L, tgate, tbeta, tk);
    } else {
#pragma unroll
        for (int e = 0; e < EK; ++e) { tk.q[e] = 0.f; tk.k[e] = 0.f; tk.g[e] = 1.f; }
#pragma unroll
        for (int e = 0; e < EV; ++e) tk.v[e] = 0.f;
        tk.gs = 0.f;
        tk.b = 0.f;
    }
    float x[EK], ob[EV];
    window_read<FAM, K, V, LPU>(p, h, l, gbase, sh, L, tk, x, ob);
    const bool bf16 = p.sketch_bf16;
    for (int i0 = 0; i0 < r; i0 += 32) {
        const int nr = min(32, r - i0);
        const float* cs = csm + i0 * K;
        const unsigned char* us = sh + L.ush + i0 * V * esz;
        auto loadU = [&](int i, float (&u)[EV]) {
            if (bf16) ld_bf16<EV>(reinterpret_cast<const uint16_t*>(us) + i * V + l * EV, u);
            else ld_f32<EV>(reinterpret_cast<const float*>(us) + i * V + l * EV, u);
        };
        if (nr <= 8) readout<8, K, V, LPU>(cs, nr, l, gbase, x, ob, loadU);
        else if (nr <= 16) readout<16, K, V, LPU>(cs, nr, l, gbase, x, ob, loadU);
        else readout<32, K, V, LPU>(cs, nr, l, gbase, x, ob, loadU);
    }
    if (active) st_f32<EV>(p.out + unit * V + l * EV, ob);
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
            stage_unit_bulk<FAM, K, V>(p, unit, sh, L, nullptr, 0, bar, p.stall && unit == 0 ? 16u : 0u);
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
int decode_bytes(int fam, int K, int V, int P, int rmax, int esz, int wpc) {
    return align16(rmax * K * 4) + 16 + wpc * (32 / DEC_LPU) * dec_unit_bytes(fam, K, V, P, rmax * V * esz);
}

template <int FAM, int K, int V>
cudaError_t decode_t(const StepParams& p, int rmax, cudaStream_t stream) {
    const int esz = p.sketch_bf16 ? 2 : 4;
    const int upw = 32 / DEC_LPU;
    int wpc = DEC_MAX_WARPS;
    while (wpc > 1 && (decode_bytes(FAM, K, V, p.p, rmax, esz, wpc) > SMEM_LIMIT || (wpc - 1) * upw >= p.B)) --wpc;
    const int bytes = decode_bytes(FAM, K, V, p.p, rmax, esz, wpc);
    if (bytes > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    const int upc = wpc * upw;
    const dim3 grid(unsigned((p.B + upc - 1) / upc), unsigned(p.H));
    auto kern = decode_kernel<FAM, K, V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, dim3(wpc * 32), bytes, stream>>>(p, rmax);
    return cudaGetLastError();
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
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, hpc * per_head);
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

int decode_smem_bytes(int family, int dk, int dv, int P, int rmax, int esz) {
    return decode_bytes(family, dk, dv, P, rmax, esz, 1);
}

}  // namespace ss
