// flush_mma_kernel: the Mamba-2 state-streaming kernel on the tensor cores.
//
// With a scalar decay and no erase term the window's W updates form one
// rank-W product (paper §4.1, App. B; Mamba-2 transition as in the GitHub
// page's "Overview"): in the scaled state S' = S / Gamma_j,
//     S'_W = S_0 + sum_j c_j k_j v_j^T,      c_j = b_j / Gamma_j,
// and S_W = Gamma_W S'_W.  The read-out is the product U = S_W^T Omega (and
// o = S_W^T q, project page "02 / How to Make a Sketch").  Both run as warp
// MMAs (m16n8k8, tf32 inputs, fp32 accumulation) with split-precision
// operands, x = hi + lo with hi = tf32(x): a product a*b is taken as
// a_hi*b + a_lo*b when b is exact in tf32 (bf16 values are), and as
// a_hi*b_hi + a_hi*b_lo + a_lo*b_hi otherwise, which keeps fp32 accuracy.
//
// Work split.  Persistent CTAs of 2*dv threads walk the heads.  Warp w owns
// state columns 16w .. 16w+15 for all dk rows and keeps S'^T there in MMA
// accumulator layout: lane (g = lane/4, t = lane%4) holds S'[8n+2t(+1)][16w+g(+8)]
// for every 8-row block n.  The update is S'^T += (c ⊙ V)^T K with A = the
// value columns (scaled by c_j, split) and B = the keys (exact).  Read as B
// operands with the contraction index permuted (slot t <-> row 2t, slot t+4
// <-> row 2t+1), the same accumulators feed the read-out MMA
// U^T = Omega'^T S directly, so a warp finishes its 16 columns of U without
// talking to another warp.
//
// Memory.  The state tile arrives by one bulk copy per row into rows padded
// to dv+4 floats (conflict-free fragment loads), the window by the same bulk
// copies as the CUDA-core flush.  Waits are bounded and report
// SS_DEVICE_TIMEOUT in the caller's status word.
#include <mutex>

#include "ss_mma.cuh"

namespace ss {
namespace {

template <int K, int V>
struct MS {
    static constexpr int T = 2 * V;              // threads per CTA
    static constexpr int NT = K / 8;             // 8-row blocks of the state
    static constexpr int KS = K + 8;             // padded key / basis row (floats)
};

// Per-CTA shared-memory layout (byte offsets).
struct MmaLayout {
    int tile, kraw, vraw, sg, tq, braw, kt, pt, sc, meta, bars, total;
};

// n updates (ring + token), rows of [Omega | q] padded to e16 (a multiple of 16).
__host__ __device__ inline MmaLayout mma_layout(int K, int V, int n, int e16) {
    const int n4 = (n + 3) & ~3, nj = (n + 7) & ~7;
    MmaLayout L;
    int o = 0;
    L.tile = o; o += K * V * 4;                  // 1024-byte aligned (swizzle atom)
    L.kraw = o; o += align16(n * K * 2);
    L.vraw = o; o += align16(n * V * 2);
    L.sg = o;   o += align16(n4 * 4);
    L.tq = o;   o += align16(K * 2);
    L.braw = o; o += align16((e16 > 0 ? e16 : 1) * K * 4);
    L.kt = o;   o += align16((nj > 0 ? nj : 8) * (K + 8) * 4);
    L.pt = o;   o += align16((e16 > 0 ? e16 : 16) * (K + 8) * 4);
    L.sc = o;   o += align16((n + 1) * 16);
    L.meta = o; o += 16;
    L.bars = o; o += 16;                        // tile, window
    L.total = o + 1024;                          // room to align the base to 1024 bytes
    return L;
}

// Bytes of one head's window copies.
template <int K, int V>
__device__ __forceinline__ unsigned mma_window_bytes(const FlushParams& p, int r) {
    const int nr = p.n_ring, n4r = (nr + 3) & ~3;
    unsigned b = nr * (K * 2 + V * 2) + (nr > 0 ? n4r * 4 : 0) + r * K * 4;
    if (p.has_token) b += K * 2 + V * 2 + K * 2;
    return b;
}

// One thread: the bulk copies of head u's window (ring keys, values and
// decays, the token's key, value and query, the basis rows).
template <int K, int V>
__device__ __forceinline__ void mma_issue_window(const FlushParams& p, long long u, unsigned char* smem,
                                                 const MmaLayout& L, uint64_t* bar, unsigned extra) {
    const int h = int(u % p.H);
    const int r = p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;   // basis rows
    mbar_expect_tx(bar, mma_window_bytes<K, V>(p, r) + extra);
    const int nr = p.n_ring, n4r = (nr + 3) & ~3;
    if (nr > 0) {
        bulk_g2s(smem + L.kraw, p.ring_k + u * p.W * K, nr * K * 2, bar);
        bulk_g2s(smem + L.vraw, p.ring_v + u * p.W * V, nr * V * 2, bar);
        bulk_g2s(smem + L.sg, p.ring_gate + u * p.Wg, n4r * 4, bar);
    }
    if (p.has_token) {
        bulk_g2s(smem + L.kraw + nr * K * 2, p.tok_k + u * K, K * 2, bar);
        bulk_g2s(smem + L.vraw + nr * V * 2, p.tok_v + u * V, V * 2, bar);
        bulk_g2s(smem + L.tq, p.tok_q + u * K, K * 2, bar);
    }
    if (r > 0) bulk_g2s(smem + L.braw, p.basis + (long long)p.off[h] * K, r * K * 4, bar);
}

// Per-head preparation: widened keys kt[j][row] (zero past the window),
// the extended basis pt[e][row] = [Omega_h | q | 0 ...] and the update
// coefficients sc[j] = (b_j / Gamma_j, Gamma_j, fold factor, 0) with
// sc[n].x = Gamma_n; meta[0] = the mask of updates that fold.
template <int K, int V>
__device__ __forceinline__ void mma_prepare(const FlushParams& p, int h, int n, int r_h, int e16,
                                            unsigned char* smem, const MmaLayout& L, float tgate, int t) {
    using S = MS<K, V>;
    constexpr int T = S::T, KS = S::KS;
    const int lane = t & 31, warp = t >> 5;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(smem + L.kraw);
    const float* sg = reinterpret_cast<const float*>(smem + L.sg);
    const uint16_t* tq = reinterpret_cast<const uint16_t*>(smem + L.tq);
    const float* braw = reinterpret_cast<const float*>(smem + L.braw);
    float* kt = reinterpret_cast<float*>(smem + L.kt);
    float* pt = reinterpret_cast<float*>(smem + L.pt);
    float4* sc = reinterpret_cast<float4*>(smem + L.sc);
    unsigned* meta = reinterpret_cast<unsigned*>(smem + L.meta);

    const int nj = (n + 7) & ~7;
    for (int pc = t; pc < nj * (K / 8); pc += T) {            // 8 keys per step
        const int j = pc / (K / 8), c0 = (pc % (K / 8)) * 8;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (j < n) {
            const uint4 w = *reinterpret_cast<const uint4*>(kraw + j * K + c0);
            a = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
            b = make_float4(bf2f_lo(w.z), bf2f_hi(w.z), bf2f_lo(w.w), bf2f_hi(w.w));
        }
        *reinterpret_cast<float4*>(kt + j * KS + c0) = a;
        *reinterpret_cast<float4*>(kt + j * KS + c0 + 4) = b;
    }
    for (int pc = t; pc < e16 * (K / 4); pc += T) {           // 4 basis entries per step
        const int e = pc / (K / 4), c = (pc % (K / 4)) * 4;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < r_h) {
            val = *reinterpret_cast<const float4*>(braw + e * K + c);
        } else if (e == r_h && p.has_token) {
            const uint2 w = *reinterpret_cast<const uint2*>(tq + c);
            val = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
        }
        *reinterpret_cast<float4*>(pt + e * KS + c) = val;
    }
    if (warp == 0) {
        // lane j holds (a_j, b_j) with a_j = exp(dt_j A_h), b_j = dt_j; running
        // products by a log-step scan, or sequentially with folds when a
        // product leaves [2^-32, 2^32].
        const float A = p.A[h];
        float al = 1.f, bl = 0.f;
        if (lane < n) {
            bl = lane >= p.n_ring ? tgate : sg[lane];
            al = expf(bl * A);
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
            if (lane == 0) {
                float gam = 1.f;
                unsigned mask = 0;
                for (int j = 0; j < n; ++j) {
                    float g = gam * al_s[j], rs = 1.f;
                    if (!(g >= GAMMA_LO && g <= GAMMA_HI)) { rs = g; g = 1.f; mask |= 1u << j; }
                    gam = g;
                    sc[j] = make_float4(bl_s[j] * __frcp_rn(gam), gam, rs, 0.f);
                }
                sc[n] = make_float4(gam, 0.f, 0.f, 0.f);
                meta[0] = mask;
            }
            __syncwarp();
        }
    }
}

template <int K, int V, bool MIXED>
__global__ void __launch_bounds__(2 * V, V == 64 ? 3 : 2) flush_mma_kernel(const __grid_constant__ FlushParams p,
                                                                         const __grid_constant__ CUtensorMap tmap,
                                                                         int e16) {
    using S = MS<K, V>;
    constexpr int NT = S::NT, KS = S::KS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int g = lane >> 2, q4 = lane & 3;
    const int col = 16 * warp + g;                   // this lane's columns: col, col + 8
    const long long units = (long long)p.B * p.H;
    const int n = p.n_ring + p.has_token;
    const MmaLayout L = mma_layout(K, V, n, e16);
    const unsigned char* tile = smem + L.tile;
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(smem + L.vraw);
    const float* kt = reinterpret_cast<const float*>(smem + L.kt);
    const float* pt = reinterpret_cast<const float*>(smem + L.pt);
    const float4* sc = reinterpret_cast<const float4*>(smem + L.sc);
    const unsigned* meta = reinterpret_cast<const unsigned*>(smem + L.meta);
    uint64_t* tbar = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* wbar = tbar + 1;
    const bool stall = p.stall && blockIdx.x == 0;

    unsigned pending = 0;                            // thread 0: bit 0 tile, bit 1 window in flight
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
    if (u < units && t == 0) {
        issue_state_tile<K, V>(&tmap, u, smem + L.tile, tbar);
        mma_issue_window<K, V>(p, u, smem, L, wbar, stall ? 16u : 0u);
        pending = 3u;
    }

    bool ok = true;
    int k_fail = 0;                                   // mixed steps: the head whose wait ran out
    for (int k = 0; u < units; ++k, u = MIXED ? fq->next : u + gridDim.x) {
        const int h = int(u % p.H);
        const long long b = u / p.H;
        const float tgate = (p.has_token && warp == 0) ? p.tok_gate[u] : 0.f;
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

        // 1. S'^T in accumulator layout: acc[nb] covers rows 8 nb .. 8 nb + 7.
        //    With the swizzle the 32 lanes of each load hit 32 different banks.
        float acc[NT][4];
        {
            const int o00 = tile_off<K>(2 * q4, col), o10 = tile_off<K>(2 * q4 + 1, col);
            const int o01 = tile_off<K>(2 * q4, col + 8), o11 = tile_off<K>(2 * q4 + 1, col + 8);
#pragma unroll
            for (int nb = 0; nb < NT; ++nb) {                         // rows + 8 nb: same swizzle phase
                const unsigned char* r = tile + nb * 8 * 128;
                acc[nb][0] = *reinterpret_cast<const float*>(r + o00);
                acc[nb][1] = *reinterpret_cast<const float*>(r + o10);
                acc[nb][2] = *reinterpret_cast<const float*>(r + o01);
                acc[nb][3] = *reinterpret_cast<const float*>(r + o11);
            }
        }

        // 2. Per-head preparation.
        // dense-fallback heads keep no sketch here: dense_copy_kernel writes their state copy
        const int r_h = p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;
        const int ne = r_h + p.has_token;                             // columns of [Omega_h | q]
        mma_prepare<K, V>(p, h, n, r_h, e16, smem, L, tgate, t);
        __syncthreads();                                              // (B)

        // 3. The tile buffer is free: start the next head's state.
        {
            const long long un = MIXED ? fq->next : u + gridDim.x;
            if (un < units && t == 0) {
                issue_state_tile<K, V>(&tmap, un, smem + L.tile, tbar);
                pending |= 1u;
            }
        }

        // 4. The window's updates, 8 at a time: S'^T += A K with
        //    A[col][j] = c_j v_j[col] (split) and K[j][row] exact.
        // Updates run in segments between folds (normally one segment).
        const unsigned mask = meta[0];
        for (int j_lo = 0; j_lo < n;) {
            int j_hi = j_lo + 1;
            while (j_hi < n && !((mask >> j_hi) & 1u)) ++j_hi;
            if ((mask >> j_lo) & 1u) {
                const float f = sc[j_lo].z;
#pragma unroll
                for (int nb = 0; nb < NT; ++nb)
#pragma unroll
                    for (int s = 0; s < 4; ++s) acc[nb][s] *= f;
            }
            for (int j0 = j_lo & ~7; j0 < j_hi; j0 += 8) {
                uint32_t ah[4], al[4];
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const int j = j0 + q4 + 4 * (s >> 1);
                    const int c = col + 8 * (s & 1);
                    float a = 0.f;
                    if (j >= j_lo && j < j_hi) a = sc[j].x * bf2f(vraw[j * V + c]);
                    split_tf32(a, ah[s], al[s]);
                }
                const float* k0 = kt + (j0 + q4) * KS + g;
                // all hi products first, then all lo ones: dependent MMAs on
                // one accumulator are NT instructions apart
#pragma unroll
                for (int nb = 0; nb < NT; ++nb)
                    mma_tf32(acc[nb], ah, __float_as_uint(k0[8 * nb]), __float_as_uint(k0[4 * KS + 8 * nb]));
#pragma unroll
                for (int nb = 0; nb < NT; ++nb)
                    mma_tf32(acc[nb], al, __float_as_uint(k0[8 * nb]), __float_as_uint(k0[4 * KS + 8 * nb]));
            }
            j_lo = j_hi;
        }
        const float gam_n = sc[n].x;
        __syncthreads();                                              // (C) window read

        // 5. The window buffers are free: start the next head's window.
        {
            const long long un = MIXED ? fq->next : u + gridDim.x;
            if (t == 0 && un < units) {
                mma_issue_window<K, V>(p, un, smem, L, wbar, 0u);
                pending |= 2u;
            }
        }

        // 6. True state S = Gamma_n S', written back (8 consecutive columns
        //    of 4 rows per warp store).
        float* st = p.state + u * (long long)(K * V);
#pragma unroll
        for (int nb = 0; nb < NT; ++nb) {
#pragma unroll
            for (int s = 0; s < 4; ++s) acc[nb][s] *= gam_n;
            float* r0 = st + (8 * nb + 2 * q4) * V + col;
            __stcs(r0, acc[nb][0]);
            __stcs(r0 + V, acc[nb][1]);
            __stcs(r0 + 8, acc[nb][2]);
            __stcs(r0 + V + 8, acc[nb][3]);
        }

        // 7. Read-out U^T = Omega'^T S: rows e of [Omega_h | q] (16 per
        //    tile) against this warp's 16 columns, contraction over dk with
        //    the accumulators as B operands (slot t <-> row 2t, t+4 <-> 2t+1).
#pragma unroll 1
        for (int e0 = 0; e0 < ne; e0 += 16) {
            // three partial products in separate accumulators (hi*hi,
            // hi*lo, lo*hi), so consecutive MMAs are independent
            float d[3][2][4];
#pragma unroll
            for (int a = 0; a < 3; ++a)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) d[a][hf][s2] = 0.f;
#pragma unroll
            for (int nb = 0; nb < NT; ++nb) {
                const float2 x0 = *reinterpret_cast<const float2*>(pt + (e0 + g) * KS + 8 * nb + 2 * q4);
                const float2 x1 = *reinterpret_cast<const float2*>(pt + (e0 + g + 8) * KS + 8 * nb + 2 * q4);
                uint32_t ph[4], pl[4];
                split_tf32(x0.x, ph[0], pl[0]);
                split_tf32(x1.x, ph[1], pl[1]);
                split_tf32(x0.y, ph[2], pl[2]);
                split_tf32(x1.y, ph[3], pl[3]);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t bh0, bl0, bh1, bl1;
                    split_tf32_here(acc[nb][2 * half], bh0, bl0);
                    split_tf32_here(acc[nb][2 * half + 1], bh1, bl1);
                    mma_tf32(d[0][half], ph, bh0, bh1);
                    mma_tf32(d[1][half], ph, bl0, bl1);
                    mma_tf32(d[2][half], pl, bh0, bh1);
                }
            }
            // d[half]: rows e0 + g (+8), columns 16 w + 8 half + 2 t (+1)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int c = 16 * warp + 8 * half + 2 * q4;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int e = e0 + g + 8 * rr;
                    const float v0 = d[0][half][2 * rr] + (d[1][half][2 * rr] + d[2][half][2 * rr]);
                    const float v1 = d[0][half][2 * rr + 1] + (d[1][half][2 * rr + 1] + d[2][half][2 * rr + 1]);
                    if (e < r_h) {
                        const long long row = b * p.R + p.off[h] + e;
                        if (p.sketch_bf16)
                            *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.sketch) + row * V + c) =
                                uint32_t(f2bf(v0)) | (uint32_t(f2bf(v1)) << 16);
                        else
                            *reinterpret_cast<float2*>(static_cast<float*>(p.sketch) + row * V + c) =
                                make_float2(v0, v1);
                    } else if (e == r_h && p.has_token) {
                        *reinterpret_cast<float2*>(p.out + u * V + c) = make_float2(v0, v1);
                    }
                }
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

template <int K, int V, bool MIXED>
cudaError_t flush_mma_launch(const FlushParams& p, int rmax, cudaStream_t stream) {
    const int n = p.n_ring + p.has_token;
    const int e16 = (((p.do_sketch ? rmax : 0) + p.has_token) + 15) & ~15;
    const int bytes = mma_layout(K, V, n, e16).total;
    if (bytes > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    CUtensorMap map;
    cudaError_t e = state_tensor_map(p.state, (long long)p.B * p.H * K, K, V, &map);
    if (e != cudaSuccess) return e;
    auto kern = flush_mma_kernel<K, V, MIXED>;
    static KernelCache kc;
    e = ensure_smem(kern, kc, bytes);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cached_occupancy(kern, kc, MS<K, V>::T, bytes, &per_sm);
    if (e != cudaSuccess) return e;
    const long long units = (long long)p.B * p.H;
    const long long cap = (long long)per_sm * sm_count();
    const long long grid = units < cap ? units : cap;
    return launch_pdl(kern, dim3(unsigned(grid)), dim3(MS<K, V>::T), bytes, stream, p, map, e16);
}

// A mixed step (fill_in set) runs its own instance: the unit selection would
// otherwise cost the uniform kernel registers it has none to spare for.
template <int K, int V>
cudaError_t flush_mma_t(const FlushParams& p, int rmax, cudaStream_t stream) {
    return p.fill_in ? flush_mma_launch<K, V, true>(p, rmax, stream) : flush_mma_launch<K, V, false>(p, rmax, stream);
}

}  // namespace

// The driver's tensor-map encoder, fetched once through the runtime.
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled tensor_map_encoder() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(f);
    });
    return fn;
}

// Tensor map of the state viewed as (B*H*dk) rows of dv floats, boxes of
// dk rows x 32 floats, 128-byte swizzle.  The last few encodings are cached
// (the state buffer of a layer does not move between calls).
cudaError_t state_tensor_map(const float* state, long long rows, int K, int V, CUtensorMap* out, bool atom32) {
    struct Entry { int dev; const float* ptr; long long rows; int K, V; bool atom32; CUtensorMap map; };
    static Entry cache[8];
    static int next = 0, used = 0;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
        const Entry& e = cache[i];
        if (e.dev == dev && e.ptr == state && e.rows == rows && e.K == K && e.V == V && e.atom32 == atom32) {
            *out = e.map;
            return cudaSuccess;
        }
    }
    EncodeTiled enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cuuint64_t(V), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(V) * 4};
    const cuuint32_t box[2] = {32, cuuint32_t(K)};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap m;
    const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(state), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    cache[next] = Entry{dev, state, rows, K, V, atom32, m};
    next = (next + 1) % 8;
    if (used < 8) ++used;
    *out = m;
    return cudaSuccess;
}

cudaError_t launch_flush_mma(int dk, int dv, const FlushParams& p, int rmax, cudaStream_t stream) {
    if (dk == 128 && dv == 64) return flush_mma_t<128, 64>(p, rmax, stream);
    if (dk == 128 && dv == 128) return flush_mma_t<128, 128>(p, rmax, stream);
    if (dk == 64 && dv == 64) return flush_mma_t<64, 64>(p, rmax, stream);
    if (dk == 64 && dv == 128) return flush_mma_t<64, 128>(p, rmax, stream);
    return cudaErrorInvalidValue;
}

int flush_mma_smem_bytes(int dk, int dv, int n, int e16) {
    return mma_layout(dk, dv, n, e16).total;
}

}  // namespace ss
