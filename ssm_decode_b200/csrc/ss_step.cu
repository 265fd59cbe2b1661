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
// One warp serves one (sequence, head) unit; lane l owns dk/32 consecutive
// key channels and dv/32 consecutive value channels.  Everything a unit
// reads -- its live ring slots, its sketch rows and the step's token -- is
// requested with cp.async at kernel entry, so a unit waits for memory once.
// The warps of a decode CTA serve the same head for consecutive sequences,
// so the head's coefficient map C is staged once per CTA.
#include "ss_common.cuh"

namespace ss {
namespace {

constexpr int DEC_MAX_WARPS = 8;

// Per-unit shared-memory layout (byte offsets) of the staged window and token.
struct UnitSmem {
    int kraw, vraw, graw, gs, bs, ush, tq, tk, tv, tg, tsc, total;
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
    L.tsc = o;  o += 16;
    L.total = o;
    return L;
}

// Issue (lane-cooperative) cp.async copies of one unit's live ring slots
// 0..p-1 and of the step's token.
template <int FAM, int K, int V>
__device__ __forceinline__ void stage_unit(const StepParams& p, long long unit, int lane,
                                           unsigned char* sh, const UnitSmem& L) {
    const long long ring_row = unit * p.W;
    const int P = p.p;
    stage(sh + L.kraw, p.ring_k + ring_row * K, P * K * 2, lane, 32);
    stage(sh + L.vraw, p.ring_v + ring_row * V, P * V * 2, lane, 32);
    const int P4 = (P + 3) & ~3;
    if (FAM == KDA) stage(sh + L.graw, p.ring_gate + ring_row * K, P * K * 4, lane, 32);
    else stage(sh + L.gs, p.ring_gate + unit * p.Wg, P4 * 4, lane, 32);
    if (FAM != MAMBA2) stage(sh + L.bs, p.ring_beta + unit * p.Wg, P4 * 4, lane, 32);
    stage(sh + L.tq, p.tok_q + unit * K, K * 2, lane, 32);
    stage(sh + L.tk, p.tok_k + unit * K, K * 2, lane, 32);
    stage(sh + L.tv, p.tok_v + unit * V, V * 2, lane, 32);
    if (FAM == KDA) stage(sh + L.tg, p.tok_gate + unit * K, K * 4, lane, 32);
    else if (lane == 0) cp_async4(sh + L.tsc, p.tok_gate + unit);
    if (FAM != MAMBA2 && lane == 1) cp_async4(sh + L.tsc + 4, p.tok_beta + unit);
}

// N consecutive bf16 values, widened.
template <int N>
__device__ __forceinline__ void ld_bf16(const uint16_t* src, float (&dst)[N]) {
    if constexpr (N == 4) {
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
    if constexpr (N == 4) {
        const float4 f = *reinterpret_cast<const float4*>(src);
        dst[0] = f.x; dst[1] = f.y; dst[2] = f.z; dst[3] = f.w;
    } else {
        static_assert(N == 2, "unsupported width");
        const float2 f = *reinterpret_cast<const float2*>(src);
        dst[0] = f.x; dst[1] = f.y;
    }
}

template <int N>
__device__ __forceinline__ void copy_bits(uint16_t* dst, const uint16_t* src) {
    if constexpr (N == 4) *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
    else *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
}

// The step's token as this lane sees it.
template <int K, int V>
struct Tok {
    static constexpr int EK = K / 32, EV = V / 32;
    float q[EK], k[EK], v[EV], g[EK];
    float gs, b;   // scalar decay input (Mamba-2 dt, GDN a) and update strength b
};

// Append the staged token, bit for bit, at ring slot p and widen it.
template <int FAM, int K, int V>
__device__ __forceinline__ void append_token(const StepParams& p, long long unit, int lane,
                                             const unsigned char* sh, const UnitSmem& L, Tok<K, V>& tk) {
    constexpr int EK = K / 32, EV = V / 32;
    const uint16_t* tq = reinterpret_cast<const uint16_t*>(sh + L.tq) + lane * EK;
    const uint16_t* tkk = reinterpret_cast<const uint16_t*>(sh + L.tk) + lane * EK;
    const uint16_t* tv = reinterpret_cast<const uint16_t*>(sh + L.tv) + lane * EV;
    const float* tsc = reinterpret_cast<const float*>(sh + L.tsc);
    const long long slot = unit * p.W + p.p;
    copy_bits<EK>(p.ring_k + slot * K + lane * EK, tkk);
    copy_bits<EV>(p.ring_v + slot * V + lane * EV, tv);
    ld_bf16<EK>(tq, tk.q);
    ld_bf16<EK>(tkk, tk.k);
    ld_bf16<EV>(tv, tk.v);
    if (FAM == KDA) {
        ld_f32<EK>(reinterpret_cast<const float*>(sh + L.tg) + lane * EK, tk.g);
        float* gdst = p.ring_gate + slot * K + lane * EK;
        if constexpr (EK == 4) *reinterpret_cast<float4*>(gdst) = make_float4(tk.g[0], tk.g[1], tk.g[2], tk.g[3]);
        else *reinterpret_cast<float2*>(gdst) = make_float2(tk.g[0], tk.g[1]);
        tk.gs = 1.f;
    } else {
        tk.gs = tsc[0];
        if (lane == 0) p.ring_gate[unit * p.Wg + p.p] = tk.gs;
#pragma unroll
        for (int e = 0; e < EK; ++e) tk.g[e] = 1.f;
    }
    if (FAM != MAMBA2) {
        tk.b = tsc[1];
        if (lane == 0) p.ring_beta[unit * p.Wg + p.p] = tk.b;
    } else {
        tk.b = tk.gs;   // b_j = dt_j
    }
}

// Butterfly reduce-scatter of NR per-lane partial sums: afterwards lane l
// holds the warp-wide total of entry l >> (5 - log2 NR).
template <int NR>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[NR], int lane) {
    constexpr int LG = NR == 8 ? 3 : NR == 16 ? 4 : 5;
    static_assert(NR == 8 || NR == 16 || NR == 32, "NR must be 8, 16 or 32");
#pragma unroll
    for (int lev = 0; lev < LG; ++lev) {
        const int half = NR >> (lev + 1);
        const int m = 16 >> lev;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(FULL, send, m);
        }
    }
#pragma unroll
    for (int m = 16 >> LG; m >= 1; m >>= 1) v[0] += __shfl_xor_sync(FULL, v[0], m);
    return v[0];
}

// Mamba-2 window read in closed form (paper §C.1: q~ = d ⊙ q).  With no
// erase term, x_j = (prod_{i>j} a_i) q, so each buffered update's read is
// k_j . q scaled by a decay; the NR dot products are reduced together.
template <int NR, int K, int V>
__device__ __forceinline__ void sweep_mamba2(const StepParams& p, int h, int lane, const unsigned char* sh,
                                             const UnitSmem& L, const Tok<K, V>& tk, float (&x)[K / 32],
                                             float (&ob)[V / 32]) {
    constexpr int EK = K / 32, EV = V / 32;
    constexpr int SH = NR == 8 ? 2 : NR == 16 ? 1 : 0;
    const int P = p.p;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw) + lane * EK;
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw) + lane * EV;
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
    const float dots = warp_reduce_scatter<NR>(v, lane);      // lane l: k_{l >> SH} . q
    // lane j: dt_j, and the decay after update j, exp(A * sum_{i>j} dt_i)
    const float A = p.A[h];
    const float dt = lane < P ? gs[lane] : (lane == P ? tk.gs : 0.f);
    float incl = dt;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const float y = __shfl_up_sync(FULL, incl, m);
        if (lane >= m) incl += y;
    }
    const float total = __shfl_sync(FULL, incl, 31);
    const float cs = dt * expf(A * (total - incl));
    const float qs = expf(A * total);
#pragma unroll
    for (int e = 0; e < EK; ++e) x[e] = qs * tk.q[e];
#pragma unroll
    for (int e = 0; e < EV; ++e) ob[e] = 0.f;
#pragma unroll 4
    for (int j = 0; j <= P; ++j) {
        const float cj = __shfl_sync(FULL, cs, j) * __shfl_sync(FULL, dots, j << SH);
        float vj[EV];
        if (j < P) {
            ld_bf16<EV>(vraw + j * V, vj);
        } else {
#pragma unroll
            for (int e = 0; e < EV; ++e) vj[e] = tk.v[e];
        }
#pragma unroll
        for (int e = 0; e < EV; ++e) ob[e] = fmaf(cj, vj[e], ob[e]);
    }
}

// Delta-rule (and generic) window read: the sequential backward sweep.
template <int FAM, int K, int V>
__device__ __forceinline__ void sweep_seq(const StepParams& p, int h, int lane, const unsigned char* sh,
                                          const UnitSmem& L, const Tok<K, V>& tk, float (&x)[K / 32],
                                          float (&ob)[V / 32]) {
    constexpr int EK = K / 32, EV = V / 32;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sh + L.kraw) + lane * EK;
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sh + L.vraw) + lane * EV;
    const float* graw = reinterpret_cast<const float*>(sh + L.graw) + lane * EK;
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
        float kx = 0.f;
#pragma unroll
        for (int e = 0; e < EK; ++e) kx = fmaf(kj[e], x[e], kx);
        const float bsx = bj * warp_sum(kx);
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
// o += sum_i c_i u_i with the sketch rows in shared memory.
template <int NR, int K, int V>
__device__ __forceinline__ void readout(const float* csm, const unsigned char* ush, int nr, bool bf16,
                                        int lane, const float (&x)[K / 32], float (&o)[V / 32]) {
    constexpr int EK = K / 32, EV = V / 32;
    constexpr int SH = NR == 8 ? 2 : NR == 16 ? 1 : 0;
    float v[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        float acc = 0.f;
        if (i < nr) {
            float cr[EK];
            ld_f32<EK>(csm + i * K + lane * EK, cr);
#pragma unroll
            for (int e = 0; e < EK; ++e) acc = fmaf(cr[e], x[e], acc);
        }
        v[i] = acc;
    }
    const float c = warp_reduce_scatter<NR>(v, lane);
#pragma unroll 4
    for (int i = 0; i < nr; ++i) {
        const float ci = __shfl_sync(FULL, c, i << SH);
        float u[EV];
        if (bf16) ld_bf16<EV>(reinterpret_cast<const uint16_t*>(ush) + i * V + lane * EV, u);
        else ld_f32<EV>(reinterpret_cast<const float*>(ush) + i * V + lane * EV, u);
#pragma unroll
        for (int e = 0; e < EV; ++e) o[e] = fmaf(ci, u[e], o[e]);
    }
}

template <int FAM, int K, int V>
__device__ __forceinline__ void window_read(const StepParams& p, int h, int lane, const unsigned char* sh,
                                            const UnitSmem& L, const Tok<K, V>& tk, float (&x)[K / 32],
                                            float (&ob)[V / 32]) {
    if constexpr (FAM == MAMBA2) {
        const int n = p.p + 1;
        if (n <= 8) sweep_mamba2<8, K, V>(p, h, lane, sh, L, tk, x, ob);
        else if (n <= 16) sweep_mamba2<16, K, V>(p, h, lane, sh, L, tk, x, ob);
        else sweep_mamba2<32, K, V>(p, h, lane, sh, L, tk, x, ob);
    } else {
        sweep_seq<FAM, K, V>(p, h, lane, sh, L, tk, x, ob);
    }
}

// ---------------------------------------------------------------------------
// decode_kernel
// ---------------------------------------------------------------------------
template <int FAM, int K, int V>
__global__ void __launch_bounds__(DEC_MAX_WARPS * 32) decode_kernel(const __grid_constant__ StepParams p,
                                                                    int rmax) {
    constexpr int EK = K / 32, EV = V / 32;
    extern __shared__ __align__(16) unsigned char smem[];
    const int wpc = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbg = (p.B + wpc - 1) / wpc;
    const int h = blockIdx.x / nbg;
    const int b = (blockIdx.x % nbg) * wpc + warp;
    const bool active = b < p.B;
    const long long unit = (long long)b * p.H + h;
    const int esz = p.sketch_bf16 ? 2 : 4;
    const int off = p.off[h], r = p.off[h + 1] - off;
    const UnitSmem L = unit_smem(FAM, K, V, p.p, rmax * V * esz);
    float* csm = reinterpret_cast<float*>(smem);
    unsigned char* sh = smem + align16(rmax * K * 4) + warp * L.total;

    stage(csm, p.coef + (long long)off * K, r * K * 4, threadIdx.x, blockDim.x);
    if (active) {
        stage_unit<FAM, K, V>(p, unit, lane, sh, L);
        stage(sh + L.ush, static_cast<const char*>(p.sketch) + (b * (long long)p.R + off) * (V * esz),
              r * V * esz, lane, 32);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    if (!active) return;                      // whole warps; no block barrier follows

    Tok<K, V> tk;
    append_token<FAM, K, V>(p, unit, lane, sh, L, tk);
    float x[EK], ob[EV];
    window_read<FAM, K, V>(p, h, lane, sh, L, tk, x, ob);
    for (int i0 = 0; i0 < r; i0 += 32) {
        const int nr = min(32, r - i0);
        const float* cs = csm + i0 * K;
        const unsigned char* us = sh + L.ush + i0 * V * esz;
        if (nr <= 8) readout<8, K, V>(cs, us, nr, p.sketch_bf16, lane, x, ob);
        else if (nr <= 16) readout<16, K, V>(cs, us, nr, p.sketch_bf16, lane, x, ob);
        else readout<32, K, V>(cs, us, nr, p.sketch_bf16, lane, x, ob);
    }
    float* dst = p.out + unit * V + lane * EV;
    if constexpr (EV == 4) *reinterpret_cast<float4*>(dst) = make_float4(ob[0], ob[1], ob[2], ob[3]);
    else *reinterpret_cast<float2*>(dst) = make_float2(ob[0], ob[1]);
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
    return unit_smem(fam, K, V, P, 0).total + align16((K + 16) * 4) + align16(V * 4);
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
        stage_unit<FAM, K, V>(p, unit, lane, sh, L);
        cp_async_commit();
        cp_async_wait_all();
        __syncwarp();
        Tok<K, V> tk;
        append_token<FAM, K, V>(p, unit, lane, sh, L, tk);
        float x[EK], ob[EV];
        window_read<FAM, K, V>(p, h, lane, sh, L, tk, x, ob);
#pragma unroll
        for (int e = 0; e < EK; ++e) qt[kpad4<K>(lane * EK + e)] = x[e];
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
int decode_bytes(int fam, int K, int V, int P, int rmax, int esz, int wpc) {
    return align16(rmax * K * 4) + wpc * unit_smem(fam, K, V, P, rmax * V * esz).total;
}

template <int FAM, int K, int V>
cudaError_t decode_t(const StepParams& p, int rmax, cudaStream_t stream) {
    const int esz = p.sketch_bf16 ? 2 : 4;
    int wpc = DEC_MAX_WARPS;
    while (wpc > 1 && (decode_bytes(FAM, K, V, p.p, rmax, esz, wpc) > SMEM_LIMIT || wpc > p.B)) --wpc;
    const int bytes = decode_bytes(FAM, K, V, p.p, rmax, esz, wpc);
    if (bytes > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    const long long grid = (long long)p.H * ((p.B + wpc - 1) / wpc);
    auto kern = decode_kernel<FAM, K, V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(grid)), dim3(wpc * 32), bytes, stream>>>(p, rmax);
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
