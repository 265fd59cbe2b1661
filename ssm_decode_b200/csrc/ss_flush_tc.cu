// flush_tc_kernel: the GDN / KDA state-streaming kernel on the fifth-generation
// tensor cores (tcgen05, operands and accumulators in tensor memory).
//
// Per (sequence, head) it reads the fp32 dk x dv state once, applies the
// window's n buffered updates, writes the state back and reads out the sketch
// U = S_W^T Omega and the exact output o = S_W^T q of the updated state
// (paper §4.1 and App. B as summarised on the paperlayer page: one full-state
// read per window, the sketch construction fused into the update; project
// page "02 / How to Make a Sketch").  dv = 128, dk in {64, 128}, n <= 16.
//
// Chunked form of the delta rule.  With A(t, j) = a_{j+1} ... a_t (A(t, t) = 1)
// and y_t = S_0^T k_t, the GDN recurrence S_t = a_t (I - b_t k_t k_t^T) S_{t-1}
// + b_t k_t v_t^T (GitHub page "Overview"; paper §C) unrolls to
//     S_W = A(n-1,-1) S_0 + sum_j A(n-1,j) k_j w_j^T,
//     w_t = b_t (v_t - A(t,-1) y_t - sum_{j<t} A(t,j) (k_t . k_j) w_j).
// KDA (S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T) is the same
// with per-channel products G(t,j) = a_{j+1} ⊙ ... ⊙ a_t: y_t = S_0^T (G(t,-1) ⊙ k_t),
// pair weights sum_c k_t[c] k_j[c] G(t,j)[c] and S_W = Diag(G(n-1,-1)) S_0 +
// sum_j (G(n-1,j) ⊙ k_j) w_j^T.  Every decay factor is a product of decays in
// [0, 1]: nothing overflows and the window needs no renormalisation.
//
// Read-out without a second pass over the state.  With S_W = Diag(g) S_0 +
// sum_j k^_j w~_j^T (g = A(n-1,-1) for GDN, G(n-1,-1) per channel for KDA; k^_j
// the update keys, w~_j = w_j scaled by A(n-1,j) for GDN), for any probe x (a
// basis vector omega_e or the query q):
//     S_W^T x = S_0^T (g ⊙ x) + sum_j w~_j (k^_j . x).
// One tensor-core pass over S_0 yields Y and S_0^T (g ⊙ x); the small products
// k^_j . x run on the CUDA cores meanwhile and are added by a few more MMAs
// (A = W~^T, already in TMEM for the update) onto the pass's output.
//
// Tensor-core products per head (tf32 operands, fp32 accumulators in TMEM,
// M = dv = 128 on the TMEM lanes; lane v is state column v):
//     D   = S_0^T [Y's keys | g ⊙ probes | their lo halves | (KDA) keys' lo]
//                                                        N <= 96, K = dk
//     D  += W~^T (K^ X^T) on the probe columns           N = 16 or 32, K = 16
//     C  += W~^T K^   (C = Diag(g) S_0 before)           N = dk,  K = 16
// An instruction costs about as much at N = 16 as at N = 128 (it is bound by
// reading its 128 x 8 slice of A), so products sharing an A are packed along
// N.  fp32 accuracy from tf32 operands: each fp32 operand is split x = hi + lo,
// hi = x with the low 13 mantissa bits cleared (the tensor core takes a tf32
// operand from fp32 by this truncation, so a raw fp32 value serves as its own
// hi half), lo = x - hi exactly; products are hi*hi + hi*lo + lo*hi, or
// hi*b + lo*b when b is exact in tf32 (bf16 keys and queries).  Both halves of
// S_0 live in TMEM (A operands); the B operands in 128-byte-swizzled shared
// memory (K-major: 16-byte atoms; MN-major: 32-byte atoms, the only layout the
// tensor core takes for MN-major tf32).
//
// The update accumulates onto C = Diag(g) S_0 (written by the workers from
// S_0's TMEM copy), so C ends as S_W^T itself.
//
// Work split.  Persistent CTAs, one per SM, of 8 worker warps and a control
// warp; CTA c walks heads c, c + grid, ...  Worker (v, half) owns state column
// v and half of the dk rows; lane 0 of the control warp issues every bulk copy
// and MMA, so no worker stalls while the tensor core drains its queue.  The
// state tile arrives by bulk tensor copies; once it is split into TMEM (early
// in the head) the tile buffer takes the next head's copy, which has the rest
// of the head to arrive.  A head's S_W leaves by coalesced stores from
// registers while the next head's pass runs on the tensor core, so the
// workers' wait for the stores to drain overlaps the pass.  The window
// (keys, values, decays, query, basis rows) arrives by bulk copies.  MMA
// groups complete on mbarriers.  Every wait is bounded: when one runs out the
// kernel sets SS_DEVICE_TIMEOUT in the caller's status word, waits (bounded)
// for its own copies and MMAs in flight, releases its tensor memory and
// returns.
#include "ss_mma.cuh"
#include "ss_tc.cuh"

namespace ss {
namespace {

constexpr int TV = 128;            // dv: state columns = TMEM lanes
constexpr int NWK = 256;           // worker threads: two per state column
constexpr int TT = NWK + 32;       // and the control warp
constexpr int NJ = 16;             // update slots per head (n <= 16)
// Tensor-memory columns (all 512 allocated; one CTA per SM).
constexpr uint32_t T_HI = 0;       // S_0 (its raw fp32 value, the hi half): dk columns
constexpr uint32_t T_LO = 128;     // lo half of S_0: dk columns
constexpr uint32_t T_C = 256;      // the update's accumulator C: dk columns
constexpr uint32_t T_D = 384;      // the pass over S_0: up to 96 columns
constexpr uint32_t T_WH = 480;     // hi half of W~^T: 16 columns
constexpr uint32_t T_WL = 496;     // lo half of W~^T: 16 columns
constexpr uint32_t T_COLS = 512;
// KDA heads whose running decay products fall below this take the pair
// weights channel by channel instead of through k_j / G(j,-1).
constexpr float KDA_GMIN = 7.888609052210118e-31f;   // 2^-100

// tf32 value the tensor core takes from an fp32 operand: the low 13 mantissa bits cleared.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

// Barrier of the 256 worker threads only (named barrier 1).
__device__ __forceinline__ void wsync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }
// The same, returning whether any worker passed `x` true.
__device__ __forceinline__ bool wsync_or(bool x) {
    unsigned r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"(unsigned(x))
        : "memory");
    return r != 0;
}

// Rows of the pass's B operand (K-major, 16-byte-atom swizzle, dk columns):
//   [0, 16)              Y's keys (KDA: hi half of G(t,-1) ⊙ k_t)
//   [16, 16 + E)         g ⊙ probe e, hi halves: omega_e for e < r_h, q at
//                        e = r_h (with a token), then zeros
//   [16 + E, 16 + 2E)    lo halves of the same rows
//   [16 + 2E, 32 + 2E)   KDA only: lo half of Y's keys
// E = 16 or 32 (read-out columns rounded up).  The pass with S_0's hi half
// uses every row; with its lo half the first 16 + E.
__host__ __device__ constexpr int pass_rows(int fam, int E) { return 16 + 2 * E + (fam == KDA ? 16 : 0); }

// Per-CTA shared-memory layout (byte offsets from a 1024-byte-aligned base).
struct TcLayout {
    int tile, bp, ku, ku2, kxh, kxl, kq, kp, xp, kraw, vraw, graw, braw, sg, sb, tq, tab, bars, total;
};

// Rows of the row-major buffers are padded by 16 bytes, so the rows that a
// warp reads together start in different banks.
__host__ __device__ inline TcLayout tc_layout(int fam, int K, int E) {
    const bool kda = fam == KDA;
    TcLayout L;
    int o = 0;
    L.tile = o; o += K * TV * 4;                    // state tile (32-byte-atom swizzle)
    L.bp = o;   o += pass_rows(fam, E) * K * 4;     // the pass's B operand
    L.ku = o;   o += NJ * K * 4;                    // update keys, MN-major (KDA: hi half)
    L.ku2 = o;  o += kda ? NJ * K * 4 : 0;          // KDA: their lo half
    L.kxh = o;  o += E * 128;                       // k^_j . x_e, K-major [e][j] (j < 32), hi half
    L.kxl = o;  o += E * 128;                       // and lo half
    L.kq = o;   o += kda ? NJ * (K + 4) * 4 : 0;    // KDA: k_j / G(j,-1), rows padded by 16 bytes
    L.kp = o;   o += kda ? NJ * (K + 4) * 4 : 0;    // KDA: update keys, rows padded
    L.xp = o;   o += E * (K + 4) * 4;               // the probes unscaled, rows padded
    L.kraw = o; o += NJ * K * 2;
    L.vraw = o; o += NJ * TV * 2;
    L.graw = o; o += kda ? NJ * K * 4 : 0;
    L.braw = o; o += E * K * 4;                     // basis rows of the head
    L.sg = o;   o += NJ * 4;
    L.sb = o;   o += NJ * 4;
    L.tq = o;   o += align16(K * 2);
    L.tab = o;  o += (NJ * NJ + 6 * NJ + K) * 4;
    L.bars = o; o += 64;
    L.total = o + 1024;                             // room to align the base to 1024 bytes
    return L;
}

// Tables of the recursion (floats, in L.tab): P[t][j] (pair weights times b_t),
// cy[t] (weight of y_t), cb[t] = b_t, g[j] (GDN: A(n-1, j); KDA: 1), al[t] (GDN
// decays), gw[k] (KDA: G(n-1,-1)[k]).
struct Tab {
    float *P, *cy, *cb, *g, *al, *gw;
    __device__ explicit Tab(unsigned char* base) {
        float* f = reinterpret_cast<float*>(base);
        P = f;
        cy = f + NJ * NJ;
        cb = cy + NJ;
        g = cb + NJ;
        al = g + NJ;
        gw = al + 2 * NJ;
    }
};

// Basis rows of unit u's head that its flush reads.
__device__ __forceinline__ int tc_basis_rows(const FlushParams& p, long long u) {
    const int h = int(u % p.H);
    return p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;
}

// Bytes of one head's window copies.
template <int FAM, int K>
__device__ __forceinline__ unsigned tc_window_bytes(const FlushParams& p, int r) {
    const int nr = p.n_ring, n4r = (nr + 3) & ~3;
    unsigned b = unsigned(r) * K * 4;
    if (nr > 0) {
        b += nr * (K * 2 + TV * 2) + n4r * 4;        // keys, values, betas
        b += FAM == KDA ? nr * K * 4 : n4r * 4;      // decays
    }
    if (p.has_token) b += K * 2 + TV * 2 + K * 2 + (FAM == KDA ? K * 4 : 0);
    return b;
}

// One thread: the bulk copies of head u's window.  `extra` bytes more than the
// copies deliver are expected (testing hook: the wait then runs out).
template <int FAM, int K>
__device__ __forceinline__ void tc_issue_window(const FlushParams& p, long long u, unsigned char* sm,
                                                const TcLayout& L, uint64_t* bar, unsigned extra) {
    const int r = tc_basis_rows(p, u);
    mbar_expect_tx(bar, tc_window_bytes<FAM, K>(p, r) + extra);
    const long long row = u * p.W;
    const int nr = p.n_ring, n4r = (nr + 3) & ~3;
    if (nr > 0) {
        bulk_g2s(sm + L.kraw, p.ring_k + row * K, nr * K * 2, bar);
        bulk_g2s(sm + L.vraw, p.ring_v + row * TV, nr * TV * 2, bar);
        if (FAM == KDA) bulk_g2s(sm + L.graw, p.ring_gate + row * K, nr * K * 4, bar);
        else bulk_g2s(sm + L.sg, p.ring_gate + u * p.Wg, n4r * 4, bar);
        bulk_g2s(sm + L.sb, p.ring_beta + u * p.Wg, n4r * 4, bar);
    }
    if (p.has_token) {
        bulk_g2s(sm + L.kraw + nr * K * 2, p.tok_k + u * K, K * 2, bar);
        bulk_g2s(sm + L.vraw + nr * TV * 2, p.tok_v + u * TV, TV * 2, bar);
        if (FAM == KDA) bulk_g2s(sm + L.graw + nr * K * 4, p.tok_gate + u * K, K * 4, bar);
        bulk_g2s(sm + L.tq, p.tok_q + u * K, K * 2, bar);
    }
    if (r > 0) bulk_g2s(sm + L.braw, p.basis + (long long)p.off[u % p.H] * K, r * K * 4, bar);
}

// Four consecutive channels c .. c+3 (c % 4 == 0) of row `row` of a K-major
// operand buffer with `rows` rows (16-byte-atom swizzle).
__device__ __forceinline__ float4 ld_row4(const unsigned char* buf, int rows, int row, int c) {
    return *reinterpret_cast<const float4*>(buf + tc::sw128_off(rows, row, c));
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}

template <int FAM, int K>
__global__ void __launch_bounds__(TT, 1) flush_tc_kernel(const __grid_constant__ FlushParams p,
                                                        const __grid_constant__ CUtensorMap tmap, int E) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const bool ctl = warp == NWK / 32;                                // the control warp
    const bool issuer = ctl && lane == 0;
    const int v = t & (TV - 1);                                       // a worker's state column
    const int hk = (t >> 7) & 1;                                      // which half of the dk rows
    constexpr int KH = K / 2;
    const TcLayout L = tc_layout(FAM, K, E);
    const int NB = pass_rows(FAM, E);                                 // rows of the pass's B operand
    const long long units = (long long)p.B * p.H;
    const int n = p.n_ring + p.has_token;
    constexpr int KP = K + 4;                                         // padded row of the row-major buffers
    uint64_t* tbar = reinterpret_cast<uint64_t*>(sm + L.bars);       // the tile
    uint64_t* wbar = tbar + 1;                                       // the window
    uint64_t* pbar = tbar + 2;                                       // MMA groups: the pass,
    uint64_t* cbar = tbar + 3;                                       //   the read-out's correction,
    uint64_t* ubar = tbar + 4;                                       //   the update
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tbar + 5);
    const bool stall = p.stall && blockIdx.x == 0;
    Tab tab(sm + L.tab);
    unsigned char* const tile = sm + L.tile;
    unsigned char* const bp = sm + L.bp;
    const uint16_t* kraw = reinterpret_cast<const uint16_t*>(sm + L.kraw);
    const uint16_t* vraw = reinterpret_cast<const uint16_t*>(sm + L.vraw);
    const float* graw = reinterpret_cast<const float*>(sm + L.graw);
    const float* braw = reinterpret_cast<const float*>(sm + L.braw);
    const float* sg = reinterpret_cast<const float*>(sm + L.sg);
    const float* sb = reinterpret_cast<const float*>(sm + L.sb);
    const uint16_t* tq = reinterpret_cast<const uint16_t*>(sm + L.tq);
    float* kq = reinterpret_cast<float*>(sm + L.kq);                 // KDA [NJ][KP]
    float* kp = reinterpret_cast<float*>(sm + L.kp);                 // KDA [NJ][KP]
    float* xp = reinterpret_cast<float*>(sm + L.xp);                 // [E][KP]

    if (t == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(tbar + i, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc::alloc(tmem_slot, T_COLS);
        tc::relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_q = uint32_t(32 * (warp & 3)) << 16;          // this warp's TMEM lane quarter
    griddep_wait();                                                   // the previous kernel's writes are visible
    griddep_launch_next();

    // in-flight copies and MMA groups: the issuer's (bit 0 tile, bit 1 window,
    // bits 2, 3, 4: the pass, correction and update groups) and worker 0's
    // (bit 1: a window it issued itself)
    unsigned pending = 0;
    unsigned tph = 0, wph = 0, pph = 0, cph = 0, uph = 0;
    long long u_prev = -1;                                            // the head whose S_W is still in C
    long long u = blockIdx.x;
    const long long stride = gridDim.x;
    if (issuer && u < units) {
        issue_state_tile<K, TV>(&tmap, u, tile, tbar);
        tc_issue_window<FAM, K>(p, u, sm, L, wbar, stall ? 16u : 0u);
        pending = 3u;
    }
    const uint32_t s_bp = smem_u32(bp), s_ku = smem_u32(sm + L.ku), s_ku2 = smem_u32(sm + L.ku2);
    const uint32_t s_kxh = smem_u32(sm + L.kxh), s_kxl = smem_u32(sm + L.kxl);

    bool ok = true;
    for (; u < units; u += stride) {
        const int h = int(u % p.H);
        const long long b = u / p.H;
        const int r_h = tc_basis_rows(p, u);
        const int ne = r_h + p.has_token;                              // read-out columns [Omega_h | q]
        bool fail = false, slow = false;

        float vv[NJ];                                                   // the values of this column
        if (!ctl) {
            bool w_ok = mbar_wait(tbar, tph);
            w_ok = mbar_wait(wbar, wph) && w_ok;
            fail = wsync_or(!w_ok);                                     // the same verdict for every worker
            if (t == 0 && !fail) pending &= ~2u;
        }
        if (!ctl && !fail) {
            // ---- phase 1a: S_0 into TMEM, keys, scalars -----------------------------------------
            {
                // S_0's raw value (the hi half) and its lo half, this thread's column
                // and half of the rows; the tile is in the 32-byte-atom swizzle, and
                // a warp reads one 128-byte row at a time, conflict-free
                const unsigned char* colb = tile + (v >> 5) * (K * 128) + ((lane & 7) << 2);
#pragma unroll
                for (int k0 = 0; k0 < KH; k0 += 16) {
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int kk = hk * KH + k0 + i;
                        const float x = *reinterpret_cast<const float*>(colb + kk * 128 + (((lane >> 3) ^ (kk & 3)) << 5));
                        hi[i] = __float_as_uint(x);
                        lo[i] = __float_as_uint(x - tf32_hi(x));
                    }
                    tc::st16(tmem + lane_q + T_HI + hk * KH + k0, hi);
                    tc::st16(tmem + lane_q + T_LO + hk * KH + k0, lo);
                }
            }
#pragma unroll
            for (int j = 0; j < NJ; ++j) vv[j] = (hk == 0 && j < n) ? bf2f(vraw[j * TV + v]) : 0.f;
            if (t < NJ) {                                               // b_t and the GDN decays
                float a = 1.f, bt = 0.f;
                if (t < n) {
                    const bool tok = t >= p.n_ring;
                    bt = tok ? p.tok_beta[u] : sb[t];
                    if (FAM == GDN) a = tok ? p.tok_gate[u] : sg[t];
                }
                tab.al[t] = a;
                tab.cb[t] = bt;
            }
            bool tiny = false;
            if constexpr (FAM == GDN) {
                for (int i = t; i < NJ * (K / 4); i += NWK) {
                    const int j = i / (K / 4), c = (i % (K / 4)) * 4;
                    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (j < n) {
                        const uint2 w = *reinterpret_cast<const uint2*>(kraw + j * K + c);
                        v4 = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
                    }
                    *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, j, c)) = v4;
                    *reinterpret_cast<float4*>(sm + L.ku + tc::sw32b_off(NJ, j, c)) = v4;
                }
            } else if (t < K) {
                // thread c: prefix products G(t,-1)[c] (Y's keys, k_j / G(j,-1) for the
                // pair weights), suffix products G(n-1,j)[c] (the update's keys)
                const int c = t;
                float gam = 1.f;
                for (int j = 0; j < NJ; ++j) {
                    float x = 0.f, xq = 0.f;
                    if (j < n) {
                        gam *= graw[j * K + c];
                        const float kv = bf2f(kraw[j * K + c]);
                        x = gam * kv;
                        tiny |= !(gam >= KDA_GMIN);
                        xq = kv * __frcp_rn(gam);
                    }
                    const float hi = tf32_hi(x);
                    *reinterpret_cast<float*>(bp + tc::sw128_off(NB, j, c)) = hi;
                    *reinterpret_cast<float*>(bp + tc::sw128_off(NB, 16 + 2 * E + j, c)) = x - hi;
                    kq[j * KP + c] = xq;
                }
                tab.gw[c] = gam;
                float suf = 1.f;
                for (int j = NJ - 1; j >= 0; --j) {
                    float x = 0.f;
                    if (j < n) {
                        x = suf * bf2f(kraw[j * K + c]);
                        suf *= graw[j * K + c];
                    }
                    const float hi = tf32_hi(x);
                    const uint32_t o = tc::sw32b_off(NJ, j, c);
                    *reinterpret_cast<float*>(sm + L.ku + o) = hi;
                    *reinterpret_cast<float*>(sm + L.ku2 + o) = x - hi;
                    kp[j * KP + c] = x;
                }
            }
            slow = wsync_or(tiny) && FAM == KDA;                        // the tables above are written
            // ---- phase 1b: probes, unscaled (for k^ . x) and scaled by g (for the pass) -----------
            float g1 = 1.f;
            if (FAM == GDN) {
#pragma unroll
                for (int i = 0; i < NJ; ++i) g1 *= i < n ? tab.al[i] : 1.f;
            }
            for (int idx = t; idx < E * (K / 4); idx += NWK) {
                const int e = idx / (K / 4), c = (idx % (K / 4)) * 4;
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < r_h) {
                    x = *reinterpret_cast<const float4*>(braw + e * K + c);
                } else if (e == r_h && p.has_token) {
                    const uint2 w = *reinterpret_cast<const uint2*>(tq + c);
                    x = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
                }
                *reinterpret_cast<float4*>(xp + e * KP + c) = x;
                if (FAM == KDA) x = mul4(x, *reinterpret_cast<const float4*>(tab.gw + c));
                else x = make_float4(g1 * x.x, g1 * x.y, g1 * x.z, g1 * x.w);
                const float4 hi = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
                *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, 16 + e, c)) = hi;
                *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, 16 + E + e, c)) =
                    make_float4(x.x - hi.x, x.y - hi.y, x.z - hi.z, x.w - hi.w);
            }
            tc::wait_st();
            tc::fence_proxy_async();
        }
        tc::fence_before();
        // (1) operands written, tile read; KDA's slow flag is worker 0's to pass on
        if (t == 0) reinterpret_cast<volatile int*>(tmem_slot)[1] = slow ? 1 : 0;
        if (__syncthreads_or(fail)) { ok = false; break; }
        tph ^= 1u;
        wph ^= 1u;
        slow = FAM == KDA && reinterpret_cast<volatile int*>(tmem_slot)[1] != 0;

        if (ctl) {
            if (issuer) {
                tc::fence_after();
                pending &= ~3u;
                // the tile buffer is free: the next head's tile; the window buffers
                // too, unless KDA's slow pair weights still read the raw keys and decays
                if (u + stride < units) {
                    issue_state_tile<K, TV>(&tmap, u + stride, tile, tbar);
                    pending |= 1u;
                    if (!slow) {
                        tc_issue_window<FAM, K>(p, u + stride, sm, L, wbar, 0u);
                        pending |= 2u;
                    }
                }
                // D = S_0^T [keys | probes]: the hi half against every row, the lo half against the first 16 + E
                const uint32_t id_hi = tc::idesc_tf32(TV, NB, 0, 0), id_lo = tc::idesc_tf32(TV, 16 + E, 0, 0);
#pragma unroll 1
                for (int q = 0; q < K / 8; ++q) {
                    const uint64_t bd = tc::sdesc(s_bp + (q >> 2) * (NB * 128) + (q & 3) * 32, 16, 1024, tc::LAYOUT_SW128);
                    tc::mma_ts(tmem + T_D, tmem + T_HI + 8 * q, bd, id_hi, q > 0);
                    tc::mma_ts(tmem + T_D, tmem + T_LO + 8 * q, bd, id_lo, 1);
                }
                tc::commit(pbar);
                pending |= 4u;
            }
            __syncwarp();
        } else {
            // ---- phase 2 (beside the pass): pair sums, k^_j . x_e, the recursion's tables -----------
            {
                // pair sums for j < t, two threads per pair (half the channels each)
                const int pair = t >> 1, part = t & 1;
                int tt = 1, rem = pair;
                while (rem >= tt && tt < NJ) { rem -= tt; ++tt; }
                const int j = rem;
                const bool act = pair < n * (n - 1) / 2 && !slow;
                float acc = 0.f;
                if (act) {
#pragma unroll 4
                    for (int c = part * KH; c < (part + 1) * KH; c += 4) {
                        if (FAM == KDA) {
                            const float4 x = add4(ld_row4(bp, NB, tt, c), ld_row4(bp, NB, 16 + 2 * E + tt, c));
                            acc = dot4(x, *reinterpret_cast<const float4*>(kq + j * KP + c), acc);
                        } else {
                            acc = dot4(ld_row4(bp, NB, tt, c), ld_row4(bp, NB, j, c), acc);
                        }
                    }
                }
                acc += __shfl_xor_sync(FULL, acc, 1);
                if (act && part == 0) tab.P[tt * NJ + j] = acc;        // times b_t below
            }
            if (FAM == KDA && slow) {
                // channel by channel, with the ratio G(t,j)[c] as a running product:
                // thread (j = t / 16, group cg = t % 16) over dk / 16 channels
                const int j = t >> 4, cg = t & 15;
                constexpr int CPG = K / 16;
                float acc[NJ];
#pragma unroll
                for (int q = 0; q < NJ; ++q) acc[q] = 0.f;
                if (j < n) {
                    for (int ci = 0; ci < CPG; ++ci) {
                        const int c = cg * CPG + ci;
                        const float kj = bf2f(kraw[j * K + c]);
                        float r = 1.f;
#pragma unroll
                        for (int q = 1; q < NJ; ++q) {
                            if (q > j && q < n) {
                                r *= graw[q * K + c];
                                acc[q] = fmaf(kj * bf2f(kraw[q * K + c]), r, acc[q]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < NJ; ++q) {
                    float x = acc[q];
                    x += __shfl_xor_sync(FULL, x, 1);
                    x += __shfl_xor_sync(FULL, x, 2);
                    x += __shfl_xor_sync(FULL, x, 4);
                    x += __shfl_xor_sync(FULL, x, 8);
                    acc[q] = x;
                }
                if (cg == 0 && j < n) {
#pragma unroll
                    for (int q = 0; q < NJ; ++q)
                        if (q > j && q < n) tab.P[q * NJ + j] = acc[q];
                }
            }
            // k^_j . x_e (unscaled probes): thread (j = t / 16, e = t % 16, and e + 16),
            // split into hi and lo halves as the B operand of the correction MMAs
            {
                const int j = t >> 4, e0 = t & 15;
                const float* krow = FAM == KDA ? kp + j * KP : nullptr;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int e = e0 + 16 * half;
                    if (e >= E) break;
                    float acc0 = 0.f, acc1 = 0.f;
                    if (j < n && e < ne) {
                        const float* xrow = xp + e * KP;
#pragma unroll 4
                        for (int c = 0; c < K; c += 8) {
                            float4 k0, k1;
                            if (FAM == KDA) {
                                k0 = *reinterpret_cast<const float4*>(krow + c);
                                k1 = *reinterpret_cast<const float4*>(krow + c + 4);
                            } else {
                                k0 = ld_row4(bp, NB, j, c);
                                k1 = ld_row4(bp, NB, j, c + 4);
                            }
                            acc0 = dot4(k0, *reinterpret_cast<const float4*>(xrow + c), acc0);
                            acc1 = dot4(k1, *reinterpret_cast<const float4*>(xrow + c + 4), acc1);
                        }
                    }
                    const float x = acc0 + acc1;
                    const float hi = tf32_hi(x);
                    *reinterpret_cast<float*>(sm + L.kxh + tc::sw128_off(E, e, j)) = hi;
                    *reinterpret_cast<float*>(sm + L.kxl + tc::sw128_off(E, e, j)) = x - hi;
                }
            }
            tc::fence_proxy_async();
            if (n > 0) {
                // the previous head's S_W (in C) to global memory, then C = Diag(g) S_0
                // for this head; this thread's column and half of the rows
                if (u_prev >= 0) {
                    fail = wsync_or(!mbar_wait(ubar, uph));
                    tc::fence_after();
                }
                if (!fail) {
                    float g1 = 1.f;
                    if (FAM == GDN) {
#pragma unroll
                        for (int i = 0; i < NJ; ++i) g1 *= i < n ? tab.al[i] : 1.f;
                    }
                    float* dst = p.state + u_prev * (long long)(K * TV) + v;
#pragma unroll 1
                    for (int k0 = 0; k0 < KH; k0 += 32) {
                        const int kb = hk * KH + k0;
                        uint32_t cr[2][16], sh[2][16];
                        if (u_prev >= 0) {
                            tc::ld16(tmem + lane_q + T_C + kb, cr[0]);
                            tc::ld16(tmem + lane_q + T_C + kb + 16, cr[1]);
                        }
                        tc::ld16(tmem + lane_q + T_HI + kb, sh[0]);
                        tc::ld16(tmem + lane_q + T_HI + kb + 16, sh[1]);
                        tc::wait_ld();
                        if (u_prev >= 0) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                __stcs(dst + (long long)(kb + i) * TV, __uint_as_float(cr[i >> 4][i & 15]));
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float dec = FAM == KDA ? tab.gw[kb + i] : g1;
                            sh[i >> 4][i & 15] = __float_as_uint(dec * __uint_as_float(sh[i >> 4][i & 15]));
                        }
                        tc::st16(tmem + lane_q + T_C + kb, sh[0]);
                        tc::st16(tmem + lane_q + T_C + kb + 16, sh[1]);
                    }
                    tc::wait_st();
                }
            }
            wsync();                                                    // (2) raw pair sums
            if (t == 0 && slow && u + stride < units) {                 // KDA slow path: the window now
                tc_issue_window<FAM, K>(p, u + stride, sm, L, wbar, 0u);
                pending |= 2u;
            }
            if (t < NJ) {
                const int tt = t;
                float al[NJ], pr[NJ];
#pragma unroll
                for (int i = 0; i < NJ; ++i) {
                    al[i] = tab.al[i];
                    pr[i] = tab.P[tt * NJ + i];
                }
                const float cbt = tab.cb[tt];
                if (FAM == GDN) {
                    float r = 1.f;                                      // A(tt, j) for j = tt-1 .. -1
#pragma unroll
                    for (int j = NJ - 2; j >= 0; --j) {
                        if (j < tt) {
                            r *= al[j + 1];
                            pr[j] *= cbt * r;
                        }
                    }
                    r *= al[0];
                    tab.cy[tt] = tt < n ? cbt * r : 0.f;
                    float gsuf = 1.f;                                   // A(n-1, tt)
#pragma unroll
                    for (int i = 1; i < NJ; ++i)
                        if (i > tt && i < n) gsuf *= al[i];
                    tab.g[tt] = tt < n ? gsuf : 0.f;
                } else {
#pragma unroll
                    for (int j = 0; j < NJ; ++j) pr[j] *= cbt;
                    tab.cy[tt] = tt < n ? cbt : 0.f;
                    tab.g[tt] = tt < n ? 1.f : 0.f;
                }
                if (tt < n) {
#pragma unroll
                    for (int j = 0; j < NJ - 1; ++j)
                        if (j < tt) tab.P[tt * NJ + j] = pr[j];
                }
            }
            wsync();                                                    // (3) tables

            // ---- the pass is done: Y -> w (recursion), W~ into TMEM ----------------------------
            if (!fail) fail = wsync_or(!mbar_wait(pbar, pph));
            tc::fence_after();
            if (!fail && hk == 0 && n > 0) {
                uint32_t yr[16];
                float y[16];
                tc::ld16(tmem + lane_q + T_D, yr);
                if (FAM == KDA) {
                    uint32_t yl[16];
                    tc::ld16(tmem + lane_q + T_D + 16 + 2 * E, yl);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) y[i] = __uint_as_float(yr[i]) + __uint_as_float(yl[i]);
                } else {
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) y[i] = __uint_as_float(yr[i]);
                }
                float w[NJ];
#pragma unroll
                for (int tt = 0; tt < NJ; ++tt) {
                    float x = tab.cb[tt] * vv[tt] - tab.cy[tt] * y[tt];
#pragma unroll
                    for (int j = 0; j < tt; ++j) x = fmaf(-tab.P[tt * NJ + j], w[j], x);
                    w[tt] = tt < n ? x : 0.f;
                }
                uint32_t wh[16], wl[16];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const float x = w[j] * tab.g[j];                    // w~_j
                    const float hi = tf32_hi(x);
                    wh[j] = __float_as_uint(hi);
                    wl[j] = __float_as_uint(x - hi);
                }
                tc::st16(tmem + lane_q + T_WH, wh);
                tc::st16(tmem + lane_q + T_WL, wl);
                tc::wait_st();
            }
        }
        tc::fence_before();
        if (__syncthreads_or(fail)) { ok = false; break; }              // (4) W~ and k^.x ready
        pph ^= 1u;
        if (n > 0 && u_prev >= 0) uph ^= 1u;
        if (issuer) {
            pending &= ~(4u | 16u);
            tc::fence_after();
            // the probes' correction D[:, 16 ..] += W~^T (K^ X^T), then C += W~^T K^;
            // each group completes on its own mbarrier (committed even when empty)
            const int nq = (n + 7) / 8;
            if (n > 0 && ne > 0) {
                const uint32_t id_x = tc::idesc_tf32(TV, E, 0, 0);
                for (int q = 0; q < nq; ++q) {
                    const uint64_t xh = tc::sdesc(s_kxh + q * 32, 16, 1024, tc::LAYOUT_SW128);
                    const uint64_t xl = tc::sdesc(s_kxl + q * 32, 16, 1024, tc::LAYOUT_SW128);
                    tc::mma_ts(tmem + T_D + 16, tmem + T_WH + 8 * q, xh, id_x, 1);
                    tc::mma_ts(tmem + T_D + 16, tmem + T_WH + 8 * q, xl, id_x, 1);
                    tc::mma_ts(tmem + T_D + 16, tmem + T_WL + 8 * q, xh, id_x, 1);
                }
            }
            tc::commit(cbar);
            if (n > 0) {
                const uint32_t id_u = tc::idesc_tf32(TV, K, 0, 1);
                for (int q = 0; q < nq; ++q) {
                    const uint64_t bh = tc::sdesc(s_ku + q * 1024, NJ * 128, 512, tc::LAYOUT_SW128_32B);
                    tc::mma_ts(tmem + T_C, tmem + T_WH + 8 * q, bh, id_u, 1);
                    tc::mma_ts(tmem + T_C, tmem + T_WL + 8 * q, bh, id_u, 1);
                    if (FAM == KDA)
                        tc::mma_ts(tmem + T_C, tmem + T_WH + 8 * q,
                                   tc::sdesc(s_ku2 + q * 1024, NJ * 128, 512, tc::LAYOUT_SW128_32B), id_u, 1);
                }
                tc::commit(ubar);
                pending |= 16u;
            }
            pending |= 8u;
        }
        if (!ctl) {
            fail = wsync_or(!mbar_wait(cbar, cph));
            tc::fence_after();
            // ---- read-out: S_W^T x_e = (D_hi + D_lo)[e]; this thread's half of the columns -----
            const int e0 = 16 * hk;
            if (!fail && e0 < ne) {
                uint32_t dh[16], dl[16];
                tc::ld16(tmem + lane_q + T_D + 16 + e0, dh);
                tc::ld16(tmem + lane_q + T_D + 16 + E + e0, dl);
                tc::wait_ld();
                const long long row0 = b * p.R + p.off[h];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = e0 + i;
                    if (e < ne) {
                        const float x = __uint_as_float(dh[i]) + __uint_as_float(dl[i]);
                        if (e < r_h) {
                            const long long o = (row0 + e) * TV + v;
                            if (p.sketch_bf16) static_cast<uint16_t*>(p.sketch)[o] = f2bf(x);
                            else static_cast<float*>(p.sketch)[o] = x;
                        } else {
                            p.out[u * TV + v] = x;
                        }
                    }
                }
            }
        }
        cph ^= 1u;
        tc::fence_before();
        if (__syncthreads_or(fail)) { ok = false; break; }              // (5) TMEM, tables and buffers read
        if (issuer) pending &= ~8u;
        if (n > 0) u_prev = u;
    }
    // the last head's S_W
    if (ok && n > 0 && u_prev >= 0) {
        bool f = false;
        if (!ctl) {
            f = wsync_or(!mbar_wait(ubar, uph));
            tc::fence_after();
            if (!f) {
                float* dst = p.state + u_prev * (long long)(K * TV) + v;
#pragma unroll 1
                for (int k0 = 0; k0 < KH; k0 += 16) {
                    const int kb = hk * KH + k0;
                    uint32_t cr[16];
                    tc::ld16(tmem + lane_q + T_C + kb, cr);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) __stcs(dst + (long long)(kb + i) * TV, __uint_as_float(cr[i]));
                }
            }
        }
        if (__syncthreads_or(f)) ok = false;
        else if (issuer) pending &= ~16u;
    }
    if (!ok && (issuer || t == 0)) {
        // a bounded wait ran out: report it, then wait (bounded) for this
        // thread's copies and MMAs still in flight before the memory is released
        if (issuer) report_timeout(p.status);
        if (pending & 4u) mbar_wait(pbar, pph);
        if (pending & 8u) mbar_wait(cbar, cph);
        if (pending & 16u) mbar_wait(ubar, uph);
        if (pending & 1u) mbar_wait(tbar, tph);
        if (pending & 2u) mbar_wait(wbar, wph);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 0) tc::dealloc(tmem, T_COLS);
}

// Dynamic shared memory of a launch: more than half an SM's, so that one CTA
// of this kernel holds an SM (each CTA allocates all 512 TMEM columns; a
// second CTA on the same SM would wait for them).
constexpr int TC_MIN_SMEM = SMEM_SM / 2 + 4096;

template <int FAM, int K>
cudaError_t flush_tc_launch(const FlushParams& p, int E, cudaStream_t stream) {
    int bytes = tc_layout(FAM, K, E).total;
    if (bytes > SMEM_LIMIT) return cudaErrorInvalidConfiguration;
    if (bytes < TC_MIN_SMEM) bytes = TC_MIN_SMEM;
    CUtensorMap map;
    cudaError_t e = state_tensor_map(p.state, (long long)p.B * p.H * K, K, TV, &map, true);
    if (e != cudaSuccess) return e;
    auto kern = flush_tc_kernel<FAM, K>;
    static KernelCache kc;
    e = ensure_smem(kern, kc, bytes);
    if (e != cudaSuccess) return e;
    const long long units = (long long)p.B * p.H;
    const long long cap = sm_count();                  // one CTA per SM (it holds all 512 TMEM columns)
    const long long grid = units < cap ? units : cap;
    return launch_pdl(kern, dim3(unsigned(grid)), dim3(TT), bytes, stream, p, map, E);
}

}  // namespace

// Whether a flush runs on the tensor-core kernel: GDN or KDA, dv = 128, at
// most 16 updates, at most 32 read-out columns, a uniform batch and the fixed
// coefficient map.
bool flush_tc_eligible(int family, int dk, int dv, const FlushParams& p, int rmax) {
    if (family == MAMBA2 || dv != TV || (dk != 64 && dk != 128)) return false;
    if (p.fill_in != nullptr || (p.cmap != nullptr && p.do_sketch)) return false;
    if (p.n_ring + p.has_token > NJ) return false;
    const int ne = (p.do_sketch ? rmax : 0) + p.has_token;
    return ne <= 32;
}

cudaError_t launch_flush_tc(int family, int dk, const FlushParams& p, int rmax, cudaStream_t stream) {
    const int ne = (p.do_sketch ? rmax : 0) + p.has_token;
    const int E = ne > 16 ? 32 : 16;
    if (family == GDN) return dk == 128 ? flush_tc_launch<GDN, 128>(p, E, stream) : flush_tc_launch<GDN, 64>(p, E, stream);
    if (family == KDA) return dk == 128 ? flush_tc_launch<KDA, 128>(p, E, stream) : flush_tc_launch<KDA, 64>(p, E, stream);
    return cudaErrorInvalidValue;
}

}  // namespace ss
