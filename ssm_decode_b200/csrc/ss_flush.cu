// flush_kernel: the state-streaming kernel of the SketchSSM decode path.
//
// For every (sequence, head) it reads the fp32 dk x dv state once, applies
// the window's buffered updates (ring slots, then the step's own token) in
// order, writes the state back and, fused into the same pass over the
// registers, computes the exact output S^T q and the sketch U = S^T Omega
// (paper §4.1 and App. B as summarised on the paperlayer page: one full-state
// read per window refreshes the sketch, whose construction is fused into the
// update kernel; project page "02 / How to Make a Sketch", u_i = S^T omega_i).
// One launch serves ss_prime (zero updates), ss_flush with or without a
// token, the ReplaySSM flush (no sketch) and the Standard step (one update).
//
// Work split.  The kernel is persistent: CTA c walks heads c, c + gridDim.x,
// ...  A head is held by 2*dv threads, dv/4 column groups x 8 row blocks;
// each thread keeps a (dk/8) x 4 tile as fp32 pairs of adjacent columns, so
// tile loads/stores are 16-byte accesses and every update is a packed
// fp32x2 FMA.
//
// Memory.  One thread moves everything with bulk asynchronous copies
// (cp.async.bulk) that complete on mbarriers: the next head's state tile
// (one copy, issued once the current tile is in registers) and the next
// head's window -- keys, values, decays, query and basis rows -- issued once
// the current head's updates are done (the read-out works from its own copy
// of the basis).  Every wait is bounded: when one runs out the kernel sets
// SS_DEVICE_TIMEOUT in the caller's status word and returns.
//
// Scaled state.  Write Gamma_j for the product of the decays since the last
// fold (a scalar for Mamba-2 and GDN, a dk-vector for KDA) and keep
// S' = Diag(Gamma_j)^-1 S.  Then, with M_j and B_j = b_j k_j v_j^T:
//     w_j = S'^T (Gamma_j ⊙ k_j)                   (delta rule only)
//     d_j = b_j (v_j - w_j)                        (Mamba-2: d_j = b_j v_j)
//     S'  <- S' + (k_j ⊘ Gamma_j) d_j^T
// which is one FMA per state element for the write and one for the delta
// rule's read; the decays cost nothing per element.  Scalar decays are folded
// into the per-update coefficients instead of the keys.  When a running
// product leaves [2^-32, 2^32] the decay is folded into S' (one multiply per
// element) and the product restarts at 1; a zero decay is applied exactly so.
#include "ss_common.cuh"

namespace ss {
namespace {

// Floats of a duplicated, row-block-padded K-vector: 8 row blocks of dk/8
// channels stored as (x, x) pairs, plus 4 floats of padding per block so the
// row blocks a warp reads together fall in different banks.
__host__ __device__ constexpr int kd_len(int K) { return 8 * (2 * (K / 8) + 4); }

template <int K, int V>
struct FS {
    static constexpr int T = 2 * V;             // threads per CTA
    static constexpr int R = K / 8;             // state rows per thread
    static constexpr int KB = 2 * R + 4;        // floats per row block of a duplicated K-vector
    static constexpr int KD = kd_len(K);
};

// Per-CTA shared-memory layout (byte offsets).  The window (keys, values,
// decays, query and basis rows of one head) is refilled for the next head
// as soon as the current head's updates are done; the read-out then works
// from pt, the extended basis [Omega_h | q | 0 ...] built from it.
struct FlushLayout {
    int tile, kraw, vraw, graw, sg, sb, tq, braw;
    int kd, ku, fin, sc, pt, meta, bars, total;
};

__host__ __device__ inline FlushLayout flush_layout(int fam, int K, int V, int n, int rpad) {
    const int KD = kd_len(K);
    const int n4 = (n + 3) & ~3;
    FlushLayout L;
    int o = 0;
    L.tile = o; o += align16(K * V * 4);
    L.kraw = o; o += align16(n * K * 2);
    L.vraw = o; o += align16(n * V * 2);
    L.graw = o; o += align16(fam == KDA ? n * K * 4 : 0);
    L.sg = o;   o += align16(fam == KDA ? 0 : n4 * 4);
    L.sb = o;   o += align16(fam == MAMBA2 ? 0 : n4 * 4);
    L.tq = o;   o += align16(K * 2);
    L.braw = o; o += align16(rpad * K * 4);
    L.kd = o;   o += align16(n * KD * 4);
    L.ku = o;   o += align16(fam == KDA ? n * KD * 4 : 0);
    L.fin = o;  o += align16(fam == KDA ? KD * 4 : 0);
    L.sc = o;   o += align16((n + 1) * 16);
    L.pt = o;   o += align16(rpad * K * 4);
    L.meta = o; o += 16;
    L.bars = o; o += 16;                        // tile, window
    L.total = o;
    return L;
}

// Index of channel c's duplicated pair in a row-block-padded K-vector.
template <int K>
__device__ __forceinline__ int kdup(int c) {
    constexpr int R = K / 8;
    return (c / R) * (2 * R + 4) + (c % R) * 2;
}

// Bytes of one head's window copies (what the window mbarrier expects).
template <int FAM, int K, int V>
__device__ __forceinline__ unsigned window_bytes(const FlushParams& p, int r) {
    const int n4r = (p.n_ring + 3) & ~3;
    unsigned b = p.n_ring * (K * 2 + V * 2) + r * K * 4;
    if (FAM == KDA) b += p.n_ring * K * 4;
    else if (p.n_ring > 0) b += n4r * 4;
    if (FAM != MAMBA2 && p.n_ring > 0) b += n4r * 4;
    if (p.has_token) b += K * 2 + V * 2 + K * 2 + (FAM == KDA ? K * 4 : 0);
    return b;
}

// Issue (one thread) the bulk copies of head u's window.
template <int FAM, int K, int V>
__device__ __forceinline__ void issue_window(const FlushParams& p, long long u, unsigned char* base,
                                             const FlushLayout& L, uint64_t* bar, unsigned extra) {
    const int h = int(u % p.H);
    const int r = p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;   // basis rows
    mbar_expect_tx(bar, window_bytes<FAM, K, V>(p, r) + extra);
    const long long ring_row = u * p.W;
    const int nr = p.n_ring, n4r = (nr + 3) & ~3;
    if (nr > 0) {
        bulk_g2s(base + L.kraw, p.ring_k + ring_row * K, nr * K * 2, bar);
        bulk_g2s(base + L.vraw, p.ring_v + ring_row * V, nr * V * 2, bar);
        if (FAM == KDA) bulk_g2s(base + L.graw, p.ring_gate + ring_row * K, nr * K * 4, bar);
        else bulk_g2s(base + L.sg, p.ring_gate + u * p.Wg, n4r * 4, bar);
        if (FAM != MAMBA2) bulk_g2s(base + L.sb, p.ring_beta + u * p.Wg, n4r * 4, bar);
    }
    if (p.has_token) {
        bulk_g2s(base + L.kraw + nr * K * 2, p.tok_k + u * K, K * 2, bar);
        bulk_g2s(base + L.vraw + nr * V * 2, p.tok_v + u * V, V * 2, bar);
        if (FAM == KDA) bulk_g2s(base + L.graw + nr * K * 4, p.tok_gate + u * K, K * 4, bar);
        bulk_g2s(base + L.tq, p.tok_q + u * K, K * 2, bar);
    }
    if (r > 0) bulk_g2s(base + L.braw, p.basis + (long long)p.off[h] * K, r * K * 4, bar);
}

// Sequential decay scan with folds, one warp, channels lane + 32 m
// (the slow path; used when some running product leaves the range).
template <int FAM, int K>
__device__ void scan_with_folds(int n, int n_ring, const float* al_in, const float* bl_in,
                                const uint16_t* kraw, const float* graw, float* kd, float* ku,
                                float* fin, float4* sc, unsigned* meta, int lane) {
    constexpr int CPL = K / 32;
    float gam[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) gam[m] = 1.f;
    unsigned mask = 0;
    for (int j = 0; j < n; ++j) {
        const float bj = bl_in[j];
        float g[CPL];
        bool need = false;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            const float a = (FAM == KDA) ? graw[j * K + lane + 32 * m] : al_in[j];
            g[m] = gam[m] * a;
            need |= !(g[m] >= GAMMA_LO && g[m] <= GAMMA_HI);
        }
        const bool fold = __any_sync(FULL, need);
        if (FAM == KDA) {
#pragma unroll
            for (int m = 0; m < CPL; ++m) {
                const int c = lane + 32 * m;
                const float kv = bf2f(kraw[j * K + c]);
                float2* kdp = reinterpret_cast<float2*>(kd + j * kd_len(K) + kdup<K>(c));
                float2* kup = reinterpret_cast<float2*>(ku + j * kd_len(K) + kdup<K>(c));
                if (fold) {            // ku carries the fold vector; Gamma_j = 1
                    *kup = dup2(g[m]);
                    *kdp = dup2(kv);
                    gam[m] = 1.f;
                } else {
                    gam[m] = g[m];
                    *kdp = dup2(g[m] * kv);
                    *kup = dup2(kv * __frcp_rn(g[m]));
                }
            }
            if (lane == 0) sc[j] = make_float4(bj, 1.f, 0.f, 0.f);
        } else {
            float rs = 1.f;
            if (fold) { rs = g[0]; gam[0] = 1.f; }
            else gam[0] = g[0];
            if (lane == 0) sc[j] = make_float4(bj * __frcp_rn(gam[0]), gam[0], rs, 0.f);
        }
        if (fold) mask |= 1u << j;
    }
    if (FAM == KDA) {
#pragma unroll
        for (int m = 0; m < CPL; ++m)
            *reinterpret_cast<float2*>(fin + kdup<K>(lane + 32 * m)) = dup2(gam[m]);
    } else if (lane == 0) {
        sc[n] = make_float4(gam[0], 0.f, 0.f, 0.f);
    }
    if (lane == 0) meta[0] = mask;
}


// Per-head preparation (phase 2): duplicated keys (and for KDA the scaled
// keys and their scan), the scalar-decay coefficients, and the rows of the
// extended basis [Omega_h | q | 0 ...] after the basis rows.  Returns nothing;
// sc[], kd[], ku[], fin[] and meta[0] are written for the update loop.
template <int FAM, int K, int V>
__device__ __forceinline__ void prepare_head(const FlushParams& p, int h, int n, int r_h, int rpad,
                                             unsigned char* slot, const FlushLayout& L,
                                             unsigned char* smem, float tgate, float tbeta, int t) {
    using S = FS<K, V>;
    constexpr int T = S::T, KD = S::KD, R = S::R;
    const int lane = t & 31, warp = t >> 5;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(slot + L.kraw);
    const float* graw = reinterpret_cast<const float*>(slot + L.graw);
    const float* sg = reinterpret_cast<const float*>(slot + L.sg);
    const float* sb = reinterpret_cast<const float*>(slot + L.sb);
    const uint16_t* tq = reinterpret_cast<const uint16_t*>(slot + L.tq);
    const float* braw = reinterpret_cast<const float*>(slot + L.braw);
    float* pt = reinterpret_cast<float*>(smem + L.pt);
    float* kd = reinterpret_cast<float*>(smem + L.kd);
    float* ku = reinterpret_cast<float*>(smem + L.ku);
    float* fin = reinterpret_cast<float*>(smem + L.fin);
    float4* sc = reinterpret_cast<float4*>(smem + L.sc);
    unsigned* meta = reinterpret_cast<unsigned*>(smem + L.meta);

    // the extended basis [Omega_h | q | 0 ...], rpad rows of dk floats
    for (int idx = t * 4; idx < rpad * K; idx += T * 4) {
        const int e = idx / K, c = idx % K;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < r_h) {
            val = *reinterpret_cast<const float4*>(braw + idx);
        } else if (e == r_h && p.has_token) {
            const uint2 w = *reinterpret_cast<const uint2*>(tq + c);
            val = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
        }
        *reinterpret_cast<float4*>(pt + idx) = val;
    }

    if (FAM != KDA) {
        // duplicated keys, 8 channels (one 16-byte row piece) per step; the 8
        // channels of a piece lie in one row block (dk/8 >= 8)
        static_assert(R % 8 == 0, "row blocks of whole 8-channel pieces");
        for (int pc = t; pc < n * (K / 8); pc += T) {
            const int j = pc / (K / 8), c0 = (pc % (K / 8)) * 8;
            const uint4 w = *reinterpret_cast<const uint4*>(kraw + j * K + c0);
            float4* d = reinterpret_cast<float4*>(kd + j * KD + kdup<K>(c0));
            const float k0 = bf2f_lo(w.x), k1 = bf2f_hi(w.x), k2 = bf2f_lo(w.y), k3 = bf2f_hi(w.y);
            const float k4 = bf2f_lo(w.z), k5 = bf2f_hi(w.z), k6 = bf2f_lo(w.w), k7 = bf2f_hi(w.w);
            d[0] = make_float4(k0, k0, k1, k1);
            d[1] = make_float4(k2, k2, k3, k3);
            d[2] = make_float4(k4, k4, k5, k5);
            d[3] = make_float4(k6, k6, k7, k7);
        }
        if (warp == 0) {
            // scalar decays: lane j holds (a_j, b_j); running products by a
            // log-step scan; folds only if a product leaves the range.
            float al = 1.f, bl = 0.f;
            if (lane < n) {
                const bool tok = lane >= p.n_ring;
                const float g = tok ? tgate : sg[lane];
                if (FAM == MAMBA2) { bl = g; al = expf(g * p.A[h]); }
                else { al = g; bl = tok ? tbeta : sb[lane]; }
            }
            float G = al;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float y = __shfl_up_sync(FULL, G, m);
                if (lane >= m) G *= y;
            }
            const bool out = lane < n && !(G >= GAMMA_LO && G <= GAMMA_HI);
            if (!__any_sync(FULL, out)) {
                if (lane < n) sc[lane] = make_float4(bl * __frcp_rn(G), G, 1.f, 0.f);
                const float Gn = __shfl_sync(FULL, G, n > 0 ? n - 1 : 0);
                if (lane == 0) { sc[n] = make_float4(n > 0 ? Gn : 1.f, 0.f, 0.f, 0.f); meta[0] = 0u; }
            } else {
                __shared__ float al_s[SS_MAX_WINDOW], bl_s[SS_MAX_WINDOW];
                al_s[lane] = al;
                bl_s[lane] = bl;
                __syncwarp();
                scan_with_folds<FAM, K>(n, p.n_ring, al_s, bl_s, kraw, graw, kd, ku, fin, sc, meta, lane);
            }
        }
    } else {
        bool bad = false;
        if (t < K) {                                          // one channel per thread
            const int c = t;
            const int pc = kdup<K>(c);
            float gam = 1.f;
            for (int j = 0; j < n; ++j) {
                const float g = gam * graw[j * K + c];
                bad |= !(g >= GAMMA_LO && g <= GAMMA_HI);
                gam = g;
                const float kv = bf2f(kraw[j * K + c]);
                *reinterpret_cast<float2*>(kd + j * KD + pc) = dup2(g * kv);
                *reinterpret_cast<float2*>(ku + j * KD + pc) = dup2(kv * __frcp_rn(g));
            }
            *reinterpret_cast<float2*>(fin + pc) = dup2(gam);
        }
        const int any_bad = __syncthreads_or(bad);
        if (warp == 0 && lane < n) {
            const float bl = lane >= p.n_ring ? tbeta : sb[lane];
            if (!any_bad) sc[lane] = make_float4(bl, 1.f, 0.f, 0.f);
        }
        if (any_bad && warp == 0) {
            __shared__ float bl_s[SS_MAX_WINDOW];
            bl_s[lane] = lane < n ? (lane >= p.n_ring ? tbeta : sb[lane]) : 0.f;
            __syncwarp();
            scan_with_folds<FAM, K>(n, p.n_ring, nullptr, bl_s, kraw, graw, kd, ku, fin, sc, meta, lane);
        } else if (warp == 0 && lane == 0) {
            meta[0] = 0u;
        }
    }
}

// Whether the coefficient map of a rank-r head fits the flush's scratch: the
// tile buffer (dk x dv floats) holds U (r rows of dv + 4 floats; the pad puts
// consecutive rows on different banks), then per-warp partial sums of at least
// one map row (dv/16 warps x dk) and later the Gram matrix (r x r).
__host__ __device__ constexpr int umap_stride(int V) { return V + 4; }
__host__ __device__ inline bool map_fits(int K, int V, int r) {
    const int free_floats = K * V - r * umap_stride(V);
    return r <= V && free_floats >= (V / 16) * K && free_floats >= r * r;
}

// The low-rank-plus-diagonal map's scratch in the tile buffer (floats):
// column energies (V), the pivots (4 ints, padded to 16), the pivot columns
// L (4 x dk), the diagonal d (dk), per-warp partials of d ((dv/16) x dk),
// P^T L (r x 4), then the Gram matrix (r x r).
constexpr int LRD_PIV = 4;
__host__ __device__ inline int lrd_g_offset(int K, int V, int r) {
    return V + 16 + LRD_PIV * K + K + (V / 16) * K + LRD_PIV * r;
}
__host__ __device__ inline bool lrd_map_fits(int K, int V, int r) {
    return r <= K && lrd_g_offset(K, V, r) + r * r <= K * V;
}

// The low-rank-plus-diagonal map's Z and Gram matrix (paper §A.2.2, read as
// in the oracle's coefficient_map_lrd): the state metric H = S S^T is replaced
// by H^ = L L^T + diag(d), L = the LRD_PIV output columns of S with the most
// energy ||S[:, v]||^2 (ties to the lower column), d[k] = the energy of row k
// in the other columns.  With P the head's basis (rows in the extended-basis
// buffer, as P^T):
//     Z = P^T H^ = (P^T L) L^T + P^T diag(d)       (r x dk, in place over P^T)
//     G = P^T H^ P = (P^T L)(P^T L)^T + P^T diag(d) P
// from the updated state (this thread's R x 4 tile in `st`), with no pass over
// HBM.  Returns G's address in the tile buffer.
template <int K, int V>
__device__ __forceinline__ float* lrd_metric(const FlushParams& p, const float2 (&st)[K / 8][2], int r,
                                             unsigned char* smem, const FlushLayout& L, int t) {
    using S = FS<K, V>;
    constexpr int T = S::T, R = S::R, NW = T / 32;
    const int lane = t & 31, warp = t >> 5;
    const int cgw = lane & 3, rb = lane >> 2;
    const int c0 = warp * 16 + cgw * 4, row0 = rb * R;
    float* energy = reinterpret_cast<float*>(smem + L.tile);   // [V]
    int* piv = reinterpret_cast<int*>(energy + V);             // [LRD_PIV]
    float* lcol = energy + V + 16;                             // [LRD_PIV][K]
    float* dg = lcol + LRD_PIV * K;                            // [K]
    float* dpart = dg + K;                                     // [NW][K]
    float* pl = dpart + NW * K;                                // [r][LRD_PIV]
    float* g = energy + lrd_g_offset(K, V, r);                 // [r][r]
    float* pt = reinterpret_cast<float*>(smem + L.pt);         // [r][K]: P^T, then Z
    const auto elem = [&](int i, int c) { return (c & 1) ? st[i][c >> 1].y : st[i][c >> 1].x; };

    // column energies: this thread's rows, then the sum over the row blocks
    float en[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < R; i += 2) {
            s0 = fmaf(elem(i, c), elem(i, c), s0);
            s1 = fmaf(elem(i + 1, c), elem(i + 1, c), s1);
        }
        float x = s0 + s1;
        x += __shfl_xor_sync(FULL, x, 4);
        x += __shfl_xor_sync(FULL, x, 8);
        x += __shfl_xor_sync(FULL, x, 16);
        en[c] = x;
    }
    if (rb == 0) *reinterpret_cast<float4*>(energy + c0) = make_float4(en[0], en[1], en[2], en[3]);
    __syncthreads();
    // the pivots: LRD_PIV rounds of a warp arg-max (the lower column on ties)
    if (warp == 0) {
        float ev[V / 32];
#pragma unroll
        for (int j = 0; j < V / 32; ++j) ev[j] = energy[lane + 32 * j];
        for (int q = 0; q < LRD_PIV; ++q) {
            float bv = -INFINITY;
            int bi = V;
#pragma unroll
            for (int j = 0; j < V / 32; ++j)
                if (ev[j] > bv) { bv = ev[j]; bi = lane + 32 * j; }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                const float ov = __shfl_xor_sync(FULL, bv, m);
                const int oi = __shfl_xor_sync(FULL, bi, m);
                if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if (lane == 0) piv[q] = bi;
#pragma unroll
            for (int j = 0; j < V / 32; ++j)
                if (lane + 32 * j == bi) ev[j] = -INFINITY;
        }
    }
    __syncthreads();
    int pv[LRD_PIV];
#pragma unroll
    for (int q = 0; q < LRD_PIV; ++q) pv[q] = piv[q];
    // L (the pivot columns) and this warp's part of d (the other columns' energy per row)
    float dr[R];
#pragma unroll
    for (int i = 0; i < R; ++i) dr[i] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        int q = -1;
#pragma unroll
        for (int qq = 0; qq < LRD_PIV; ++qq)
            if (pv[qq] == c0 + c) q = qq;
        if (q >= 0) {
#pragma unroll
            for (int i = 0; i < R; ++i) lcol[q * K + row0 + i] = elem(i, c);
        } else {
#pragma unroll
            for (int i = 0; i < R; ++i) dr[i] = fmaf(elem(i, c), elem(i, c), dr[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
        dr[i] += __shfl_xor_sync(FULL, dr[i], 1);
        dr[i] += __shfl_xor_sync(FULL, dr[i], 2);
    }
    if (cgw == 0) {
#pragma unroll
        for (int i = 0; i < R; ++i) dpart[warp * K + row0 + i] = dr[i];
    }
    __syncthreads();
    for (int k = t; k < K; k += T) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) s += dpart[w * K + k];
        dg[k] = s;
    }
    // P^T L
    for (int idx = t; idx < r * LRD_PIV; idx += T) {
        const int e = idx / LRD_PIV, q = idx - e * LRD_PIV;
        const float* pe = pt + e * K;
        const float* lq = lcol + q * K;
        float s0 = 0.f, s1 = 0.f;
        for (int k = 0; k < K; k += 2) {
            s0 = fmaf(pe[k], lq[k], s0);
            s1 = fmaf(pe[k + 1], lq[k + 1], s1);
        }
        pl[idx] = s0 + s1;
    }
    __syncthreads();
    // G = (P^T L)(P^T L)^T + P^T diag(d) P
    for (int idx = t; idx < r * r; idx += T) {
        const int e = idx / r, f = idx - e * r;
        if (f > e) continue;
        const float* pe = pt + e * K;
        const float* pf = pt + f * K;
        float s0 = 0.f, s1 = 0.f;
        for (int k = 0; k < K; k += 2) {
            s0 = fmaf(pe[k] * dg[k], pf[k], s0);
            s1 = fmaf(pe[k + 1] * dg[k + 1], pf[k + 1], s1);
        }
        float s = s0 + s1;
#pragma unroll
        for (int q = 0; q < LRD_PIV; ++q) s = fmaf(pl[e * LRD_PIV + q], pl[f * LRD_PIV + q], s);
        g[e * r + f] = s;
        g[f * r + e] = s;
    }
    __syncthreads();
    // Z = (P^T L) L^T + P^T diag(d), in place over P^T
    for (int idx = t; idx < r * K; idx += T) {
        const int e = idx / K, k = idx - e * K;
        float z = pt[idx] * dg[k];
#pragma unroll
        for (int q = 0; q < LRD_PIV; ++q) z = fmaf(pl[e * LRD_PIV + q], lcol[q * K + k], z);
        pt[idx] = z;
    }
    return g;
}

// State-dependent coefficient map of one head (project page, "Per window ·
// Flush: Sketch & coefficient map"; paper §A.2.1):
//     C = (U^T U + lambda I)^-1 U^T S^T,  lambda = ridge * tr(U^T U) / r,
// from the updated state S (this thread's R x 4 tile in `st`) and the sketch
// U as stored (r x dv in the tile buffer, written by the read-out).  No
// second pass over HBM: the state is still in registers.
//   1. Z = U^T S^T (r x dk): each thread contracts its 4 columns, a 2-level
//      reduce-scatter over the 4 column lanes leaves R/4 rows per lane, and
//      the dv/16 warps' partials are summed through shared memory, EC rows
//      of Z at a time.  Z lands in the extended-basis buffer (free now).
//   2. M = U^T U + lambda I in the tile buffer; warp 0 inverts it in place
//      (Gauss-Jordan, one column per lane: the row updates of a step are
//      independent, unlike the dependent chains of a Cholesky solve).
//   3. Thread k forms column k of C = M^-1 Z with independent accumulators
//      and stores it in the sketch dtype.  A pivot that is not positive and
//      finite zeroes the head's map and sets SS_DEVICE_SINGULAR_MAP.
template <int K, int V>
__device__ __forceinline__ void build_map(const FlushParams& p, const float2 (&st)[K / 8][2], int r,
                                          long long b, int h, unsigned char* smem, const FlushLayout& L,
                                          int t) {
    using S = FS<K, V>;
    constexpr int T = S::T, R = S::R, NW = T / 32;
    const int lane = t & 31, warp = t >> 5;
    const int cgw = lane & 3, rb = lane >> 2;
    const int c0 = warp * 16 + cgw * 4, row0 = rb * R;
    const int b0 = cgw & 1, b1 = (cgw >> 1) & 1;
    constexpr int US = umap_stride(V);
    float* umap = reinterpret_cast<float*>(smem + L.tile);     // [r][US]
    float* zp = umap + r * US;                                 // [EC][NW][K], then G [r][r]
    float* zs = reinterpret_cast<float*>(smem + L.pt);         // [r][K]: P, then Z, then C
    __shared__ int map_ok;
    __syncthreads();                                           // (D) U written, basis rows read
    float* g = zp;
    if (p.lrd) {
        g = lrd_metric<K, V>(p, st, r, smem, L, t);
    } else {
    const int EC = min(r, (K * V - r * US) / (NW * K));

    // 1. Z = U^T S^T
    for (int e0 = 0; e0 < r; e0 += EC) {
        const int ne = min(EC, r - e0);
        for (int el0 = 0; el0 < ne; el0 += 2) {              // two map rows per pass
            float z[2][R];
#pragma unroll
            for (int d = 0; d < 2; ++d) {
                const int el = min(el0 + d, ne - 1);
                const float4 uu = *reinterpret_cast<const float4*>(umap + (e0 + el) * US + c0);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    float2 pp = fmul2(st[i][0], make_float2(uu.x, uu.y));
                    pp = ffma2(st[i][1], make_float2(uu.z, uu.w), pp);
                    z[d][i] = pp.x + pp.y;
                }
            }
            float z2[2][R / 2];                                // lane bit 0: which half of the rows
#pragma unroll
            for (int d = 0; d < 2; ++d)
#pragma unroll
                for (int i = 0; i < R / 2; ++i) {
                    const float keep = b0 ? z[d][i + R / 2] : z[d][i], send = b0 ? z[d][i] : z[d][i + R / 2];
                    z2[d][i] = keep + __shfl_xor_sync(FULL, send, 1);
                }
            float z4[2][R / 4];                                // lane bit 1: which quarter
#pragma unroll
            for (int d = 0; d < 2; ++d)
#pragma unroll
                for (int i = 0; i < R / 4; ++i) {
                    const float keep = b1 ? z2[d][i + R / 4] : z2[d][i], send = b1 ? z2[d][i] : z2[d][i + R / 4];
                    z4[d][i] = keep + __shfl_xor_sync(FULL, send, 2);
                }
#pragma unroll
            for (int d = 0; d < 2; ++d) {
                if (el0 + d >= ne) break;
                float* dst = zp + ((el0 + d) * NW + warp) * K + row0 + b0 * (R / 2) + b1 * (R / 4);
#pragma unroll
                for (int i = 0; i < R / 4; ++i) dst[i] = z4[d][i];
            }
        }
        __syncthreads();
        for (int idx = t; idx < ne * K; idx += T) {
            const int el = idx / K, k = idx - el * K;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) sum += zp[(el * NW + w) * K + k];
            zs[(e0 + el) * K + k] = sum;
        }
        __syncthreads();
    }

    // 2. M = U^T U
    for (int idx = t; idx < r * r; idx += T) {
        const int e = idx / r, f = idx - e * r;
        if (f > e) continue;
        const float* ue = umap + e * US;
        const float* uf = umap + f * US;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;       // four independent chains
#pragma unroll 4
        for (int v = 0; v < V; v += 4) {
            const float4 a = *reinterpret_cast<const float4*>(ue + v);
            const float4 c = *reinterpret_cast<const float4*>(uf + v);
            s0 = fmaf(a.x, c.x, s0);
            s1 = fmaf(a.y, c.y, s1);
            s2 = fmaf(a.z, c.z, s2);
            s3 = fmaf(a.w, c.w, s3);
        }
        const float sum = (s0 + s1) + (s2 + s3);
        g[e * r + f] = sum;
        g[f * r + e] = sum;
    }
    }
    // M + lambda I, inverted in place by warp 0
    __syncthreads();
    if (warp == 0) {
        float tr = 0.f;
        for (int e = lane; e < r; e += 32) tr += g[e * r + e];
        const float lam = p.ridge * warp_sum(tr) / float(r);
        __syncwarp();
        for (int e = lane; e < r; e += 32) g[e * r + e] += lam;
        __syncwarp();
        // Gauss-Jordan without pivoting (M is symmetric positive definite, so
        // every pivot is a positive Schur complement); lane c owns column c.
        bool good = true;
        for (int j = 0; j < r; ++j) {
            const float piv = g[j * r + j];
            good = piv > 0.f && piv < INFINITY;                // the same value in every lane
            if (!good) break;
            const float pinv = 1.f / piv;
            __syncwarp();
            for (int c = lane; c < r; c += 32)
                if (c != j) g[j * r + c] *= pinv;              // row j
            __syncwarp();
            for (int c = lane; c < r; c += 32) {               // rows i != j, columns c != j
                if (c == j) continue;
                const float mjc = g[j * r + c];
                for (int i0 = 0; i0 < r; i0 += 8) {            // 8 rows' loads ahead of their stores
                    float mij[8], mic[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int i = min(i0 + q, r - 1);
                        mij[q] = g[i * r + j];
                        mic[q] = g[i * r + c];
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int i = i0 + q;
                        if (i < r && i != j) g[i * r + c] = fmaf(-mij[q], mjc, mic[q]);
                    }
                }
            }
            __syncwarp();
            for (int i = lane; i < r; i += 32)                 // column j last
                g[i * r + j] = i == j ? pinv : -g[i * r + j] * pinv;
            __syncwarp();
        }
        if (lane == 0) {
            map_ok = good;
            if (!good && p.status != nullptr) atomicOr(p.status, SS_DEVICE_SINGULAR_MAP);
        }
    }
    __syncthreads();

    // 3. C = M^-1 Z, one column of dk per thread, four map rows at a time,
    //    stored straight to HBM in the sketch dtype
    const bool good = map_ok != 0;
    const long long row = b * p.R + p.off[h];
    for (int k = t; k < K; k += T) {
        for (int e0 = 0; e0 < r; e0 += 4) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (good) {
                const float* m0 = g + min(e0, r - 1) * r;
                const float* m1 = g + min(e0 + 1, r - 1) * r;
                const float* m2 = g + min(e0 + 2, r - 1) * r;
                const float* m3 = g + min(e0 + 3, r - 1) * r;
                for (int f = 0; f < r; ++f) {
                    const float z = zs[f * K + k];
                    acc[0] = fmaf(m0[f], z, acc[0]);
                    acc[1] = fmaf(m1[f], z, acc[1]);
                    acc[2] = fmaf(m2[f], z, acc[2]);
                    acc[3] = fmaf(m3[f], z, acc[3]);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (e0 + q >= r) break;
                const long long o = (row + e0 + q) * K + k;
                if (p.sketch_bf16) static_cast<uint16_t*>(p.cmap)[o] = f2bf(acc[q]);
                else static_cast<float*>(p.cmap)[o] = acc[q];
            }
        }
    }
}

template <int FAM, int K, int V, bool MIXED, bool MAP>
__global__ void __launch_bounds__(2 * V, V == 64 ? 3 : 2) flush_kernel(const __grid_constant__ FlushParams p, int rpad) {
    using S = FS<K, V>;
    constexpr int R = S::R, KB = S::KB, KD = S::KD;
    extern __shared__ __align__(16) unsigned char smem[];

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int cgw = lane & 3, rb = lane >> 2;
    const int c0 = warp * 16 + cgw * 4;          // first of this thread's 4 columns
    const int row0 = rb * R;                     // first of this thread's R rows
    const long long units = (long long)p.B * p.H;
    const int n = p.n_ring + p.has_token;
    const FlushLayout L = flush_layout(FAM, K, V, n, rpad);
    const float* tile = reinterpret_cast<const float*>(smem + L.tile);
    const float* kd = reinterpret_cast<const float*>(smem + L.kd);
    const float* ku = reinterpret_cast<const float*>(smem + L.ku);
    const float* fin = reinterpret_cast<const float*>(smem + L.fin);
    const float4* sc = reinterpret_cast<const float4*>(smem + L.sc);
    const unsigned* meta = reinterpret_cast<const unsigned*>(smem + L.meta);
    uint64_t* tbar = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* wbar = tbar + 1;                   // the window
    const bool stall = p.stall && blockIdx.x == 0;

    // Only thread 0 issues copies; it tracks which barriers have copies in flight.
    unsigned pending = 0;                        // bit 0: tile, bit 1: window
    __shared__ FlushQueue fq_s;                      // mixed steps only
    FlushQueue* const fq = &fq_s;
    long long u = blockIdx.x;
    if (t == 0) {
        mbar_init(tbar, 1);
        mbar_init(wbar, 1);
        fence_mbar_init();
        if (MIXED) fq_init(fq);
    }
    __syncthreads();
    griddep_wait();                                   // the previous kernel's writes are visible
    griddep_launch_next();
    if constexpr (MIXED) {
        if (warp == 0) fq_next(p, fq, units);
        __syncthreads();
        u = fq->next;
    }
    if (t == 0 && u < units) {
        mbar_expect_tx(tbar, K * V * 4);
        bulk_g2s(smem + L.tile, p.state + u * (long long)(K * V), K * V * 4, tbar);
        issue_window<FAM, K, V>(p, u, smem, L, wbar, stall ? 16u : 0u);
        pending = 1u | 2u;
    }

    bool ok = true;
    int k_fail = 0;                                   // mixed steps: the head whose wait ran out
    for (int k = 0; u < units; ++k, u = MIXED ? fq->next : u + gridDim.x) {
        const int h = int(u % p.H);
        const long long b = u / p.H;
        float tgate = 0.f, tbeta = 0.f;                           // the token's scalar inputs
        if (p.has_token && warp == 0) {
            if (FAM != KDA) tgate = p.tok_gate[u];
            if (FAM != MAMBA2) tbeta = p.tok_beta[u];
        }
        bool w_ok = mbar_wait(tbar, k & 1);
        w_ok = mbar_wait(wbar, k & 1) && w_ok;
        if (__syncthreads_or(!w_ok)) {                              // (A) head u staged
            ok = false;
            if (MIXED) k_fail = k;
            break;
        }
        if constexpr (MIXED) {
            // After (A) every thread has read the previous q->next: queue the next unit.
            if (warp == 0) fq_next(p, fq, units);
        }
        if (t == 0) pending = 0;
        unsigned char* sl = smem;

        // 1. This thread's tile, pairs of adjacent columns.
        float2 st[R][2];
        {
            const float* tb = tile + row0 * V + c0;
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float4 a = *reinterpret_cast<const float4*>(tb + i * V);
                st[i][0] = make_float2(a.x, a.y);
                st[i][1] = make_float2(a.z, a.w);
            }
        }

        // 2. Per-head preparation: keys, decays, coefficients, extended basis.
        // dense-fallback heads keep no sketch here: dense_copy_kernel writes their state copy
        const int r_h = p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;
        const int next = r_h + p.has_token;                           // columns of [Omega_h | q]
        const int nch = (next + 3) / 4;
        prepare_head<FAM, K, V>(p, h, n, r_h, rpad, sl, L, smem, tgate, tbeta, t);
        __syncthreads();                                              // (B)

        // 3. The tile buffer is free: start the next head's state (with the
        //    coefficient map the buffer is scratch until the map is built).
        if constexpr (!MAP) {
            const long long un = MIXED ? fq->next : u + gridDim.x;
            if (t == 0 && un < units) {
                mbar_expect_tx(tbar, K * V * 4);
                bulk_g2s(smem + L.tile, p.state + un * (long long)(K * V), K * V * 4, tbar);
                pending |= 1u;
            }
        }

        // 4. Apply the updates.
        const unsigned mask = meta[0];
        const float* kdb = kd + rb * KB;
        const float* kub = ku + rb * KB;
        const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sl + L.vraw);
        auto update = [&](int j, float4 scj) {
            float2 kv[R];
#pragma unroll
            for (int i = 0; i < R; i += 2) {
                const float4 f = *reinterpret_cast<const float4*>(kdb + j * KD + 2 * i);
                kv[i] = make_float2(f.x, f.y);
                kv[i + 1] = make_float2(f.z, f.w);
            }
            float2 w2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (FAM != MAMBA2) {
                float2 w2b[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int i = 0; i < R; i += 2)
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp) {
                        w2[cp] = ffma2(kv[i], st[i][cp], w2[cp]);
                        w2b[cp] = ffma2(kv[i + 1], st[i + 1][cp], w2b[cp]);
                    }
#pragma unroll
                for (int cp = 0; cp < 2; ++cp) {
                    w2[cp] = make_float2(w2[cp].x + w2b[cp].x, w2[cp].y + w2b[cp].y);
#pragma unroll
                    for (int m = 4; m <= 16; m <<= 1) {
                        w2[cp].x += __shfl_xor_sync(FULL, w2[cp].x, m);
                        w2[cp].y += __shfl_xor_sync(FULL, w2[cp].y, m);
                    }
                }
            }
            const uint2 vv = *reinterpret_cast<const uint2*>(vraw + j * V + c0);
            const float2 v01 = make_float2(bf2f_lo(vv.x), bf2f_hi(vv.x));
            const float2 v23 = make_float2(bf2f_lo(vv.y), bf2f_hi(vv.y));
            float2 d2[2];
            if (FAM == MAMBA2) {
                d2[0] = fmul2(dup2(scj.x), v01);
                d2[1] = fmul2(dup2(scj.x), v23);
            } else {
                const float2 ncw = dup2(FAM == GDN ? -scj.y : -1.f);
                d2[0] = fmul2(dup2(scj.x), ffma2(ncw, w2[0], v01));
                d2[1] = fmul2(dup2(scj.x), ffma2(ncw, w2[1], v23));
            }
            if (FAM == KDA && !((mask >> j) & 1u)) {
#pragma unroll
                for (int i = 0; i < R; i += 2) {
                    const float4 f = *reinterpret_cast<const float4*>(kub + j * KD + 2 * i);
                    kv[i] = make_float2(f.x, f.y);
                    kv[i + 1] = make_float2(f.z, f.w);
                }
            }
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int cp = 0; cp < 2; ++cp) st[i][cp] = ffma2(kv[i], d2[cp], st[i][cp]);
        };
        if (mask == 0) {                                              // no folds (the common case)
            constexpr int UNR = V == 64 ? 2 : 1;                      // dv = 128 has no registers to spare
#pragma unroll UNR
            for (int j = 0; j < n; ++j) update(j, sc[j]);
        } else {
            for (int j = 0; j < n; ++j) {
                const float4 scj = sc[j];
                if ((mask >> j) & 1u) {
                    if (FAM == KDA) {
#pragma unroll
                        for (int i = 0; i < R; i += 2) {
                            const float4 f = *reinterpret_cast<const float4*>(kub + j * KD + 2 * i);
#pragma unroll
                            for (int cp = 0; cp < 2; ++cp) {
                                st[i][cp] = fmul2(st[i][cp], make_float2(f.x, f.y));
                                st[i + 1][cp] = fmul2(st[i + 1][cp], make_float2(f.z, f.w));
                            }
                        }
                    } else {
                        const float2 f = dup2(scj.z);
#pragma unroll
                        for (int i = 0; i < R; ++i)
#pragma unroll
                            for (int cp = 0; cp < 2; ++cp) st[i][cp] = fmul2(st[i][cp], f);
                    }
                }
                update(j, scj);
            }
        }
        __syncthreads();                                              // (C) window read

        // 5. The window buffers are free: start the next head's window.
        {
            const long long un = MIXED ? fq->next : u + gridDim.x;
            if (t == 0 && un < units) {
                issue_window<FAM, K, V>(p, un, smem, L, wbar, 0u);
                pending |= 2u;
            }
        }

        // 6. True state S = Diag(Gamma) S', written back.
        if (FAM == KDA) {
            const float* g = fin + rb * KB;
#pragma unroll
            for (int i = 0; i < R; i += 2) {
                const float4 f = *reinterpret_cast<const float4*>(g + 2 * i);
#pragma unroll
                for (int cp = 0; cp < 2; ++cp) {
                    st[i][cp] = fmul2(st[i][cp], make_float2(f.x, f.y));
                    st[i + 1][cp] = fmul2(st[i + 1][cp], make_float2(f.z, f.w));
                }
            }
        } else {
            const float2 f = dup2(sc[n].x);
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int cp = 0; cp < 2; ++cp) st[i][cp] = fmul2(st[i][cp], f);
        }
        float* sto = p.state + u * (long long)(K * V) + row0 * V + c0;
#pragma unroll
        for (int i = 0; i < R; ++i)
            __stcs(reinterpret_cast<float4*>(sto + i * V), make_float4(st[i][0].x, st[i][0].y, st[i][1].x, st[i][1].y));

        // 7. Fused read-out against [Omega_h | q], 4 basis columns per pass; a
        //    3-level reduce-scatter over the row blocks leaves row block
        //    (b2 b1 b0) with basis column 4 ch + 2 b2 + b1 for the state
        //    columns c0 + 2 b0, c0 + 2 b0 + 1.
        const float* pt = reinterpret_cast<const float*>(smem + L.pt);
        const int hb2 = (rb >> 2) & 1, hb1 = (rb >> 1) & 1, hb0 = rb & 1;
        for (int ch = 0; ch < nch; ++ch) {
            float2 acc[4][2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[e][0] = acc[e][1] = make_float2(0.f, 0.f);
                const float* prow = pt + (ch * 4 + e) * K + row0;
#pragma unroll
                for (int i = 0; i < R; i += 4) {
                    const float4 pv = *reinterpret_cast<const float4*>(prow + i);
                    const float pe[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                        for (int cp = 0; cp < 2; ++cp) acc[e][cp] = ffma2(dup2(pe[ii]), st[i + ii][cp], acc[e][cp]);
                }
            }
            float v8[2][4];                      // level 1 (lane bit 4 = rb bit 2): basis columns {0,1} | {2,3}
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float2 lo0 = acc[e][0], lo1 = acc[e][1], hi0 = acc[e + 2][0], hi1 = acc[e + 2][1];
                const float mine[4] = {hb2 ? hi0.x : lo0.x, hb2 ? hi0.y : lo0.y, hb2 ? hi1.x : lo1.x, hb2 ? hi1.y : lo1.y};
                const float give[4] = {hb2 ? lo0.x : hi0.x, hb2 ? lo0.y : hi0.y, hb2 ? lo1.x : hi1.x, hb2 ? lo1.y : hi1.y};
#pragma unroll
                for (int c = 0; c < 4; ++c) v8[e][c] = mine[c] + __shfl_xor_sync(FULL, give[c], 16);
            }
            float v4[4];                         // level 2 (lane bit 3 = rb bit 1)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float send = hb1 ? v8[0][c] : v8[1][c];
                const float keep = hb1 ? v8[1][c] : v8[0][c];
                v4[c] = keep + __shfl_xor_sync(FULL, send, 8);
            }
            float v2[2];                         // level 3 (lane bit 2 = rb bit 0): state columns
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float send = hb0 ? v4[c] : v4[c + 2];
                const float keep = hb0 ? v4[c + 2] : v4[c];
                v2[c] = keep + __shfl_xor_sync(FULL, send, 4);
            }
            const int e = ch * 4 + hb2 * 2 + hb1;
            const int col = c0 + hb0 * 2;
            if (e < r_h) {
                const long long row = b * p.R + p.off[h] + e;
                float2 us = make_float2(v2[0], v2[1]);                // U as stored
                if (p.sketch_bf16) {
                    const uint16_t h0 = f2bf(v2[0]), h1 = f2bf(v2[1]);
                    *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.sketch) + row * V + col) =
                        uint32_t(h0) | (uint32_t(h1) << 16);
                    us = make_float2(bf2f(h0), bf2f(h1));
                } else {
                    *reinterpret_cast<float2*>(static_cast<float*>(p.sketch) + row * V + col) = us;
                }
                if (MAP) *reinterpret_cast<float2*>(reinterpret_cast<float*>(smem + L.tile) + e * umap_stride(V) + col) = us;
            } else if (e == r_h && p.has_token) {
                *reinterpret_cast<float2*>(p.out + u * V + col) = make_float2(v2[0], v2[1]);
            }
        }
        if constexpr (MAP) {
            if (r_h > 0) build_map<K, V>(p, st, r_h, b, h, smem, L, t);
            __syncthreads();                                          // (E) scratch read
            // 3'. The tile buffer is free again: start the next head's state.
            const long long un = MIXED ? fq->next : u + gridDim.x;
            if (t == 0 && un < units) {
                mbar_expect_tx(tbar, K * V * 4);
                bulk_g2s(smem + L.tile, p.state + un * (long long)(K * V), K * V * 4, tbar);
                pending |= 1u;
            }
        }
    }
    if (!ok && t == 0) {                                              // a bounded wait ran out
        report_timeout(p.status);
        const int k_last = MIXED ? k_fail : int((u - blockIdx.x) / gridDim.x);   // the head whose wait failed
        if (pending & 1u) mbar_wait(tbar, k_last & 1);                // own copies: one more bounded wait
        if (pending & 2u) mbar_wait(wbar, k_last & 1);
    }
}

template <int FAM, int K, int V, bool MIXED, bool MAP>
cudaError_t flush_launch(const FlushParams& p, int rmax, cudaStream_t stream) {
    const int n = p.n_ring + p.has_token;
    const int rpad = ((p.do_sketch ? rmax : 0) + p.has_token + 3) & ~3;
    const int bytes = flush_layout(FAM, K, V, n, rpad).total;
    if (bytes > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    if (MAP && !(p.lrd ? lrd_map_fits(K, V, rmax) : map_fits(K, V, rmax))) return cudaErrorInvalidConfiguration;
    auto kern = flush_kernel<FAM, K, V, MIXED, MAP>;
    static KernelCache kc;
    cudaError_t e = ensure_smem(kern, kc, bytes);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cached_occupancy(kern, kc, FS<K, V>::T, bytes, &per_sm);
    if (e != cudaSuccess) return e;
    const long long units = (long long)p.B * p.H;
    const long long cap = (long long)per_sm * sm_count();
    const long long grid = units < cap ? units : cap;
    return launch_pdl(kern, dim3(unsigned(grid)), dim3(FS<K, V>::T), bytes, stream, p, rpad);
}

// A mixed step (fill_in set) runs its own instance, so the uniform kernel
// carries no unit selection.
template <int FAM, int K, int V>
cudaError_t flush_t(const FlushParams& p, int rmax, cudaStream_t stream) {
    if (p.cmap && p.do_sketch)
        return p.fill_in ? flush_launch<FAM, K, V, true, true>(p, rmax, stream)
                         : flush_launch<FAM, K, V, false, true>(p, rmax, stream);
    return p.fill_in ? flush_launch<FAM, K, V, true, false>(p, rmax, stream)
                     : flush_launch<FAM, K, V, false, false>(p, rmax, stream);
}

}  // namespace

// Mamba-2 runs on the warp-MMA kernel (ss_flush_mma.cu); GDN and KDA with
// dv = 128 and up to 16 updates on the tcgen05 kernel (ss_flush_tc.cu); the
// other shapes, mixed-phase steps and every family when the flush also builds
// the state-dependent coefficient map, on the CUDA-core kernel above.
cudaError_t launch_flush(int family, int dk, int dv, const FlushParams& p, int rmax, cudaStream_t stream) {
    if (family == MAMBA2 && !(p.cmap && p.do_sketch)) return launch_flush_mma(dk, dv, p, rmax, stream);
    if (flush_tc_eligible(family, dk, dv, p, rmax)) return launch_flush_tc(family, dk, p, rmax, stream);
    SS_DISPATCH(flush_t, p, rmax, stream);
}

bool flush_map_fits(int dk, int dv, int r) { return map_fits(dk, dv, r); }
bool flush_lrd_fits(int dk, int dv, int r) { return lrd_map_fits(dk, dv, r); }

namespace {

// The dense-fallback heads of a launch (project page and paper App. D:
// such heads read a BF16 copy of their state at non-flush steps).
struct DenseList {
    int n;
    int16_t head[SS_MAX_HEADS];
};

// After a flush has written the state: copy each dense head's state into its
// sketch rows, row k = S[k][:], in the sketch dtype.  Block (i, b) copies
// head dl.head[i] of sequence b; in a mixed step only flushing sequences.
template <int K, int V>
__global__ void __launch_bounds__(256) dense_copy_kernel(const __grid_constant__ FlushParams p,
                                                         const __grid_constant__ DenseList dl) {
    const int h = dl.head[blockIdx.x];
    const long long b = blockIdx.y;
    if (p.fill_in != nullptr && p.fill_in[b] != p.W - 1) return;
    const float4* src = reinterpret_cast<const float4*>(p.state + (b * p.H + h) * (long long)(K * V));
    const long long row0 = b * p.R + p.off[h];
    for (int i = threadIdx.x; i < K * V / 4; i += blockDim.x) {
        const float4 a = src[i];
        const int k = (4 * i) / V, v = (4 * i) % V;
        const long long o = (row0 + k) * V + v;
        if (p.sketch_bf16)
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.sketch) + o) =
                make_uint2(uint32_t(f2bf(a.x)) | (uint32_t(f2bf(a.y)) << 16),
                           uint32_t(f2bf(a.z)) | (uint32_t(f2bf(a.w)) << 16));
        else
            *reinterpret_cast<float4*>(static_cast<float*>(p.sketch) + o) = a;
    }
}

template <int K, int V>
cudaError_t dense_copy_t(const FlushParams& p, const DenseList& dl, cudaStream_t stream) {
    dense_copy_kernel<K, V><<<dim3(unsigned(dl.n), unsigned(p.B)), dim3(256), 0, stream>>>(p, dl);
    return cudaGetLastError();
}

}  // namespace

// Launch dense_copy_kernel for the dense heads of p.dense (none: nothing).
cudaError_t launch_dense_copy(int dk, int dv, const FlushParams& p, cudaStream_t stream) {
    DenseList dl;
    dl.n = 0;
    for (int h = 0; h < p.H; ++h)
        if (head_dense(p.dense, h)) dl.head[dl.n++] = int16_t(h);
    if (dl.n == 0 || !p.do_sketch) return cudaSuccess;
    if (dk == 128 && dv == 128) return dense_copy_t<128, 128>(p, dl, stream);
    if (dk == 128 && dv == 64) return dense_copy_t<128, 64>(p, dl, stream);
    if (dk == 64 && dv == 128) return dense_copy_t<64, 128>(p, dl, stream);
    return dense_copy_t<64, 64>(p, dl, stream);
}

// rpad = rows of [Omega | q] rounded up to 4 (the CUDA-core kernel's read-out
// passes); smap: the flush builds the state-dependent map (CUDA-core kernel).
int flush_smem_bytes(int family, int dk, int dv, int n, int rpad, bool smap) {
    if (family == MAMBA2 && !smap) return flush_mma_smem_bytes(dk, dv, n, (rpad + 15) & ~15);
    return flush_layout(family, dk, dv, n, rpad).total;
}

}  // namespace ss
