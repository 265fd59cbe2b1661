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
// pair weights sum_c k_t[c] k_j[c] G(t,j)[c] = (G(t,-1) ⊙ k_t) . (k_j / G(j,-1))
// and S_W = Diag(G(n-1,-1)) S_0 + sum_j (G(n-1,j) ⊙ k_j) w_j^T.  Every decay
// factor is a product of decays in [0, 1]: nothing overflows and the window
// needs no renormalisation (KDA heads whose products fall below 2^-100 take
// their pair weights channel by channel instead of through k_j / G(j,-1)).
//
// Read-out without a second pass over the state.  With S_W = Diag(g) S_0 +
// sum_j k^_j w~_j^T (g = A(n-1,-1) for GDN, G(n-1,-1) per channel for KDA; k^_j
// the update keys, w~_j = w_j scaled by A(n-1,j) for GDN), for any probe x (a
// basis vector omega_e or the query q):
//     S_W^T x = S_0^T (g ⊙ x) + sum_j w~_j (k^_j . x),
// and for KDA k^_j . x = (k_j / G(j,-1)) . (g ⊙ x).
//
// Tensor-core products per head (fp32 accumulators in TMEM):
//     Gm = [keys | probes] K'^T     M = 128, N = 16 (GDN) or 32 (KDA) --
//          the pair weights and k^_j . x, for the recursion and the read-out.
//          GDN in bf16: K' = the keys (exact in bf16), each probe in three
//          bf16 parts that sum to it exactly, K = 16 an instruction.  KDA in
//          tf32: K' = k_j / G(j,-1), hi and lo, against the pass's B rows
//     D  = S_0^T [keys | probes | their lo halves]   M = dv, N <= 96, K = dk
//     Dc = W~^T (K^ X^T)                              M = dv, N = 16 or 32, K = 16
//     C += W~^T K^   (C = Diag(g) S_0 before)         M = dv, N = dk, K = 16
// D, Dc and C have lane v = state column v; C ends as S_W^T.  An instruction
// costs about as much at N = 16 as at N = 128 (about 82 cycles with A in
// TMEM, 93 with A in shared memory, measured at M = 128), so products that
// share an A operand are packed along N.
// fp32 accuracy from tf32 operands: each fp32 operand is split x = hi + lo,
// hi = x with the low 13 mantissa bits cleared (the tensor core takes a tf32
// operand from fp32 by this truncation, so a raw fp32 value serves as its own
// hi half), lo = x - hi exactly; products are hi*hi + hi*lo + lo*hi, or
// hi*b + lo*b when b is exact in tf32 (bf16 keys and queries).  Both halves of
// S_0 live in TMEM (A operands); B operands in 128-byte-swizzled shared memory
// (K-major: 16-byte atoms; MN-major: 32-byte atoms, the only layout the tensor
// core takes for MN-major tf32).
//
// Work split.  Persistent CTAs, one per SM, of 8 worker warps, an issuing warp
// and a moving warp; CTA c walks heads c, c + grid, ...  Worker (v, half) owns
// state column v and half of the dk rows.  Lane 0 of the issuing warp issues
// every MMA; lane 0 of the moving warp every bulk copy in and out.  The three
// roles are paced by mbarriers only: the workers arrive (256 arrivals) when
// the keys and probes are staged, when S_0 is in TMEM and when W~ is, and the
// issuer waits for those before Gm, the pass and the correction and update;
// MMA groups complete on mbarriers the workers wait for.  The mover issues a
// head's window once phase 1 of the previous head has read the window buffers
// (fetching the scalars each copy needs a head ahead).  The workers move a
// head's tile into TMEM early in the head; its buffer then stages the
// previous head's S_W (read from C), which the mover stores before it loads
// the next head's tile into the same buffer; the read-out is staged in shared
// memory and stored the same way.  No worker
// waits for the issuer, and no one for the tensor core's queue or for stores
// to drain.  Every wait on an mbarrier is bounded: when one runs out the
// kernel sets SS_DEVICE_TIMEOUT in the caller's status word, waits (bounded)
// for its own copies and MMAs in flight, releases its tensor memory and
// returns.
#include "ss_mma.cuh"
#include "ss_tc.cuh"

namespace ss {
namespace {

constexpr int TV = 128;            // dv: state columns = TMEM lanes
constexpr int NWK = 256;           // worker threads: two per state column
constexpr int TT = NWK + 64;       // the issuing warp and the moving warp
constexpr int NJ = 16;             // update slots per head (n <= 16)
// Tensor-memory columns (all 512 allocated; one CTA per SM).
constexpr uint32_t T_HI = 0;       // S_0 (its raw fp32 value, the hi half): dk columns; later Dc
constexpr uint32_t T_LO = 128;     // lo half of S_0: dk columns
constexpr uint32_t T_C = 256;      // Diag(g) S_0 plus the update, i.e. S_W^T: dk columns
constexpr uint32_t T_D = 384;      // the pass over S_0: up to 96 columns
constexpr uint32_t T_W = 480;      // Gm (16 or 32 columns), then W~^T: hi 16, lo 16 columns
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


// Rows of the pass's B buffer (K-major, 16-byte-atom swizzle, dk columns):
//   [0, 16)              Y's keys (KDA: hi half of G(t,-1) ⊙ k_t)
//   [16, 16 + E)         probe e, hi halves (GDN: x_e; KDA: g ⊙ x_e): omega_e
//                        for e < r_h, q at e = r_h (with a token), then zeros
//   [16 + E, 16 + 2E)    lo halves of the same rows
//   [16 + 2E, 32 + 2E)   KDA only: lo half of Y's keys
// E = 16 or 32 (read-out columns rounded up).  The pass with S_0's hi half
// uses every row; with its lo half the first 16 + E.
__host__ __device__ constexpr int pass_rows(int fam, int E) { return 16 + 2 * E + (fam == KDA ? 16 : 0); }

// Per-CTA shared-memory layout (byte offsets from a 1024-byte-aligned base).
struct TcLayout {
    int tile, bp, g16, k16, ku[2], ku2[2], kq, kxh, kxl, part, ust, kraw, vraw, graw, braw, sg, sb, tq, tab, bars, total;
};

__host__ __device__ inline TcLayout tc_layout(int fam, int K, int E) {
    const bool kda = fam == KDA;
    TcLayout L;
    int o = 0;
    L.tile = o; o += K * TV * 4;                    // the state tile (32-byte-atom swizzle), then S_W
    L.bp = o;   o += pass_rows(fam, E) * K * 4;     // the pass's B buffer
    L.g16 = o;  o += kda ? 0 : 128 * K * 2;         // GDN: Gm's A in bf16, [keys | probes in three parts]
    L.k16 = o;  o += kda ? 0 : NJ * K * 2;          // GDN: Gm's B, the keys in bf16
    for (int i = 0; i < 2; ++i) {                   // update keys, MN-major (KDA: hi half), by head parity
        L.ku[i] = o; o += NJ * K * 4;
    }
    for (int i = 0; i < 2; ++i) {                   // KDA: their lo half
        L.ku2[i] = o; o += kda ? NJ * K * 4 : 0;
    }
    L.kq = o;   o += kda ? 2 * NJ * K * 4 : 0;      // KDA: k_j / G(j,-1), K-major, hi rows then lo rows
    L.kxh = o;  o += E * 128;                       // k^_j . x_e, K-major [e][j] (j < 32), hi half
    L.kxl = o;  o += E * 128;                       // and lo half
    L.part = o; o += (2 * NJ + (kda ? 2 : 3) * E) * NJ * 4;   // pieces of the pair weights and of k^ . x
    L.ust = o;  o += E * TV * 4 + TV * 4;           // the read-out staged: sketch rows, then o
    L.kraw = o; o += NJ * K * 2;
    L.vraw = o; o += NJ * TV * 2;
    L.graw = o; o += kda ? NJ * K * 4 : 0;
    L.braw = o; o += E * K * 4;                     // basis rows of the head
    L.sg = o;   o += NJ * 4;
    L.sb = o;   o += NJ * 4;
    L.tq = o;   o += align16(K * 2);
    L.tab = o;  o += (NJ * NJ + 6 * NJ + K) * 4;
    L.bars = o; o += 128;
    L.total = o + 1024;                             // room to align the base to 1024 bytes
    return L;
}

// Tables of the recursion (floats, in L.tab): P[t][j] (pair weights times b_t),
// cy[t] (weight of y_t), cb[t] = b_t, g[j] (GDN: A(n-1, j); KDA: 1), al[t] (GDN
// decays), gw[k] (KDA: G(n-1,-1)[k]).
struct Tab {
    float *P, *cy, *cb, *g, *al, *tok, *gw;
    int* hr;
    __device__ explicit Tab(unsigned char* base) {
        float* f = reinterpret_cast<float*>(base);
        P = f;
        cy = f + NJ * NJ;
        cb = cy + NJ;
        g = cb + NJ;
        al = g + NJ;
        tok = al + NJ;                                              // the next head's token b_t, a_t
        hr = reinterpret_cast<int*>(tok + 2);                       // basis rows of the head, by parity
        gw = al + 2 * NJ;
    }
};

// Basis rows of unit u's head that its flush reads, and the first of them.
__device__ __forceinline__ int tc_basis_rows(const FlushParams& p, long long u) {
    const int h = int(u % p.H);
    return p.do_sketch && !head_dense(p.dense, h) ? p.off[h + 1] - p.off[h] : 0;
}
__device__ __forceinline__ int2 tc_head_rows(const FlushParams& p, long long u) {
    return make_int2(tc_basis_rows(p, u), p.off[u % p.H]);
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

// One thread: the bulk copies of head u's window, whose basis rows hr =
// {count, first row} are given; the count is also written to *r_out for the
// threads that wait on `bar`.  `extra` bytes more than the copies deliver are
// expected (testing hook: the wait then runs out).
template <int FAM, int K>
__device__ __forceinline__ void tc_issue_window(const FlushParams& p, long long u, unsigned char* sm,
                                                const TcLayout& L, uint64_t* bar, unsigned extra, int2 hr,
                                                int* r_out) {
    const int r = hr.x;
    *r_out = r;
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
    if (r > 0) bulk_g2s(sm + L.braw, p.basis + (long long)hr.y * K, r * K * 4, bar);
}

// Bulk tensor store of one box of the state (32 columns x dk rows) from
// shared memory (bulk async-group of the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// shared -> global (bulk async-group).
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, unsigned bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// The committed stores have finished reading shared memory / are complete.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
// Four fp32 values rounded to bf16, packed in memory order.
__device__ __forceinline__ uint2 bf16x4(float4 x) {
    return make_uint2(uint32_t(f2bf(x.x)) | (uint32_t(f2bf(x.y)) << 16), uint32_t(f2bf(x.z)) | (uint32_t(f2bf(x.w)) << 16));
}
__device__ __forceinline__ float4 hi4(float4 x) { return make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w)); }

// KDA, phase 1x: thread (c, HALF) takes slots j of its half of the window.
// Prefix products G(j,-1)[c] give Y's keys (hi and lo rows of the pass's B
// buffer) and k_j / G(j,-1) (Gm's B operand, hi and lo); suffix products
// G(n-1,j)[c] the update's keys (MN-major, hi and lo).  Every load is issued
// before the products.  Returns whether a prefix product fell below KDA_GMIN.
template <int K, int HALF>
__device__ __forceinline__ bool kda_keys(int c, int n, int E, int NB, const uint16_t* kraw, const float* graw,
                                         unsigned char* bp, unsigned char* kq, unsigned char* kub,
                                         unsigned char* kub2, float* gw) {
    constexpr int J0 = HALF * (NJ / 2);
    float ga[NJ], kk[NJ / 2];
#pragma unroll
    for (int j = 0; j < NJ; ++j) ga[j] = j < n ? graw[j * K + c] : 1.f;
#pragma unroll
    for (int i = 0; i < NJ / 2; ++i) kk[i] = J0 + i < n ? bf2f(kraw[(J0 + i) * K + c]) : 0.f;
    float gam = 1.f, suf = 1.f;
#pragma unroll
    for (int j = 0; j < J0; ++j) gam *= ga[j];
#pragma unroll
    for (int j = J0 + NJ / 2; j < NJ; ++j) suf *= ga[j];
    bool tiny = false;
#pragma unroll
    for (int i = 0; i < NJ / 2; ++i) {
        const int j = J0 + i;
        gam *= ga[j];
        const bool live = j < n;
        const float x = live ? gam * kk[i] : 0.f;
        const float xq = live ? __fdividef(kk[i], gam) : 0.f;
        tiny |= live && !(gam >= KDA_GMIN);
        const float hi = tf32_hi(x), hq = tf32_hi(xq);
        *reinterpret_cast<float*>(bp + tc::sw128_off(NB, j, c)) = hi;
        *reinterpret_cast<float*>(bp + tc::sw128_off(NB, 16 + 2 * E + j, c)) = x - hi;
        *reinterpret_cast<float*>(kq + tc::sw128_off(2 * NJ, j, c)) = hq;
        *reinterpret_cast<float*>(kq + tc::sw128_off(2 * NJ, NJ + j, c)) = xq - hq;
    }
    if (HALF == 1) gw[c] = gam;
#pragma unroll
    for (int i = NJ / 2 - 1; i >= 0; --i) {
        const int j = J0 + i;
        const float x = j < n ? suf * kk[i] : 0.f;
        suf *= ga[j];
        const float hi = tf32_hi(x);
        const uint32_t o = tc::sw32b_off(NJ, j, c);
        *reinterpret_cast<float*>(kub + o) = hi;
        *reinterpret_cast<float*>(kub2 + o) = x - hi;
    }
    return tiny;
}

template <int FAM, int K>
__global__ void __launch_bounds__(TT, 1) flush_tc_kernel(const __grid_constant__ FlushParams p,
                                                        const __grid_constant__ CUtensorMap tmap, int E) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const bool ctl = warp == NWK / 32;                                // the issuing warp
    const bool mov = warp == NWK / 32 + 1;                            // the moving warp
    const bool issuer = ctl && lane == 0;                             // every MMA
    const bool mover = mov && lane == 0;                              // bulk copies in and out
    const int v = t & (TV - 1);                                       // a worker's state column
    const int hk = (t >> 7) & 1;                                      // which half of the dk rows
    constexpr int KH = K / 2;
    const TcLayout L = tc_layout(FAM, K, E);
    const int NB = pass_rows(FAM, E);                                 // rows of the pass's B buffer
    const int NG = FAM == KDA ? 32 : 16;                              // columns of Gm
    const long long units = (long long)p.B * p.H;
    const int n = p.n_ring + p.has_token;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bars);
    uint64_t* tbar = bars + 0;                                       // the tile
    uint64_t* wbar = bars + 1;                                       // the window
    uint64_t* gbar = bars + 2;                                       // MMA groups: Gm,
    uint64_t* pbar = bars + 3;                                       //   the pass,
    uint64_t* cbar = bars + 4;                                       //   the read-out's correction,
    uint64_t* ubar = bars + 5;                                       //   the update
    uint64_t* sbar = bars + 6;                                       // tile read and S_W staged (256 arrivals)
    uint64_t* rbar = bars + 7;                                       // read-out staged (256 arrivals)
    uint64_t* ebar = bars + 10;                                      // the mover's stores have read the staging buffers
    uint64_t* xbar = bars + 11;                                      // phase 1 has read the window buffers
    uint64_t* obar1 = bars + 12;                                     // workers -> issuer: keys and probes staged,
    uint64_t* obar2 = bars + 13;                                     //   S_0 in TMEM,
    uint64_t* obar5 = bars + 14;                                     //   W~ and k^.x ready (256 arrivals each)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* slow_flag = reinterpret_cast<volatile int*>(bars + 9);
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
    float* const pa = reinterpret_cast<float*>(sm + L.part);          // [NJ][NJ] from the keys' hi rows
    float* const pb = pa + NJ * NJ;                                   // [NJ][NJ] KDA: from the keys' lo rows
    float* const xa = pb + NJ * NJ;                                   // [E][NJ] from the probes' hi rows
    float* const xb = xa + E * NJ;                                    // [E][NJ] from the probes' lo rows
    float* const xc = xb + E * NJ;                                    // [E][NJ] GDN: the third bf16 part
    const size_t esz = p.sketch_bf16 ? 2 : 4;

    if (t == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(bars + i, 1);
        mbar_init(sbar, NWK);
        mbar_init(rbar, NWK);
        mbar_init(ebar, 1);
        mbar_init(xbar, 1);
        mbar_init(obar1, NWK);
        mbar_init(obar2, NWK);
        mbar_init(obar5, NWK);
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

    // MMA groups the issuer committed to gbar, pbar, cbar and ubar: before the
    // memory is released it waits (bounded) for the last of each.
    unsigned ng = 0, np = 0, nc = 0, nu = 0;
    unsigned tph = 0, wph = 0, gph = 0, pph = 0, cph = 0, uph = 0, sph = 0, rph = 0, eph = 0;
    long long u = blockIdx.x;
    const long long stride = gridDim.x;
    const uint32_t s_bp = smem_u32(bp), s_kq = smem_u32(sm + L.kq);
    const uint32_t s_kxh = smem_u32(sm + L.kxh), s_kxl = smem_u32(sm + L.kxl);

    // Workers: S_W of head `up` (in C) into the tile buffer for the mover,
    // once the update of that head has completed; arrive on sbar when done.
    auto stage_sw = [&]() -> bool {
        const bool f = wsync_or(!mbar_wait(ubar, uph));
        tc::fence_after();
        if (f) return true;
        unsigned char* colb = tile + (v >> 5) * (K * 128) + ((lane & 7) << 2);
#pragma unroll 1
        for (int k0 = 0; k0 < KH; k0 += 32) {
            const int kb = hk * KH + k0;
            uint32_t cr[2][16];
            tc::ld16(tmem + lane_q + T_C + kb, cr[0]);
            tc::ld16(tmem + lane_q + T_C + kb + 16, cr[1]);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int kk = kb + i;
                *reinterpret_cast<uint32_t*>(colb + kk * 128 + (((lane >> 3) ^ (kk & 3)) << 5)) = cr[i >> 4][i & 15];
            }
        }
        tc::fence_proxy_async();
        mbar_arrive(sbar);
        return false;
    };
    // Workers: the read-out of a head, once its correction has completed:
    // S_W^T x_e = g (D_hi + D_lo)[e] + Dc[e], staged in shared memory for the
    // mover; this thread's half of the columns.  Arrives on rbar.
    auto readout = [&](int ne_p, int r_p, float g_p) -> bool {
        // the correction is done, and the mover has read the previous read-out
        // out of the staging buffer (one arrival per mover iteration)
        const bool f = wsync_or(!mbar_wait(cbar, cph) || !mbar_wait(ebar, eph));
        eph ^= 1u;
        tc::fence_after();
        if (f) return true;
        const int e0 = 16 * hk;
        if (e0 < ne_p) {
            uint32_t dh[16], dl[16], dc[16];
            tc::ld16(tmem + lane_q + T_D + 16 + e0, dh);
            tc::ld16(tmem + lane_q + T_D + 16 + E + e0, dl);
            if (n > 0) tc::ld16(tmem + lane_q + T_HI + e0, dc);
            tc::wait_ld();
            // every sketch slot of this half is written (rows at or past r_p are
            // never copied out), so that no store sits behind a branch
            unsigned char* ust = sm + L.ust;
            float x[16], tokx = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = g_p * (__uint_as_float(dh[i]) + __uint_as_float(dl[i]));
                if (n > 0) x[i] += __uint_as_float(dc[i]);
                tokx = e0 + i == r_p ? x[i] : tokx;
            }
            if (p.sketch_bf16) {
#pragma unroll
                for (int i = 0; i < 16; ++i) reinterpret_cast<uint16_t*>(ust)[(e0 + i) * TV + v] = f2bf(x[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) reinterpret_cast<float*>(ust)[(e0 + i) * TV + v] = x[i];
            }
            if (p.has_token && r_p >= e0 && r_p < e0 + 16) reinterpret_cast<float*>(ust + E * TV * 4)[v] = tokx;
        }
        tc::fence_proxy_async();
        mbar_arrive(rbar);
        return false;
    };

    // The read-out of a head in two parts: its values from TMEM (this thread's
    // half of the columns, once the correction has completed), then, once the
    // mover has read the previous read-out out of the staging buffer, the
    // staging stores and the arrival on rbar.
    auto ro_load = [&](int ne_p, int r_p, float g_p, float (&x)[16], float& tokx) {
        const int e0 = 16 * hk;
        if (e0 >= ne_p) return;
        uint32_t dh[16], dl[16], dc[16];
        tc::ld16(tmem + lane_q + T_D + 16 + e0, dh);
        tc::ld16(tmem + lane_q + T_D + 16 + E + e0, dl);
        if (n > 0) tc::ld16(tmem + lane_q + T_HI + e0, dc);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            x[i] = g_p * (__uint_as_float(dh[i]) + __uint_as_float(dl[i]));
            if (n > 0) x[i] += __uint_as_float(dc[i]);
            tokx = e0 + i == r_p ? x[i] : tokx;
        }
    };
    auto ro_stage = [&](int ne_p, int r_p, const float (&x)[16], float tokx) {
        const int e0 = 16 * hk;
        if (e0 < ne_p) {
            // every sketch slot of this half is written (rows at or past r_p are
            // never copied out), so that no store sits behind a branch
            unsigned char* ust = sm + L.ust;
            if (p.sketch_bf16) {
#pragma unroll
                for (int i = 0; i < 16; ++i) reinterpret_cast<uint16_t*>(ust)[(e0 + i) * TV + v] = f2bf(x[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) reinterpret_cast<float*>(ust)[(e0 + i) * TV + v] = x[i];
            }
            if (p.has_token && r_p >= e0 && r_p < e0 + 16) reinterpret_cast<float*>(ust + E * TV * 4)[v] = tokx;
        }
        tc::fence_proxy_async();
        mbar_arrive(rbar);
    };

    bool ok = true;
    if (mov) {
        // ---- the moving warp: windows and tiles in; read-outs and S_W out ----------------------------
        // Per head k: once phase 1 of head k has read the window buffers, head
        // k+1's window; the read-out of head k-1 (staged early in head k), then
        // S_W of head k-1 (staged in the tile buffer once head k's tile is in
        // TMEM); once both stores have read shared memory, head k+1's tile.  The
        // scalars each copy needs (basis rows, token b_t and a_t) are fetched a
        // head ahead into registers.
        if (mover) {
            long long up = -1;
            bool tile_out = false;                                      // a tile copy in flight
            long long nwin = 0;                                         // windows issued
            int2 h_prev = make_int2(0, 0), h_cur = make_int2(0, 0), h_next = make_int2(0, 0);
            float tb_next = 0.f, tg_next = 1.f;
            auto fetch = [&](long long uu) {
                h_next = tc_head_rows(p, uu);
                if (p.has_token) {
                    tb_next = p.tok_beta[uu];
                    if (FAM == GDN) tg_next = p.tok_gate[uu];
                }
            };
            // the next head's window: its token scalars and basis rows go to
            // shared memory before the copies (the window's barrier publishes them)
            auto issue_window = [&](long long uu, long long j, unsigned extra) {
                tab.tok[0] = tb_next;
                tab.tok[1] = tg_next;
                tc_issue_window<FAM, K>(p, uu, sm, L, wbar, extra, h_next, tab.hr + (j & 1));
                ++nwin;
            };
            if (u < units) {
                issue_state_tile<K, TV>(&tmap, u, tile, tbar);
                tile_out = true;
                fetch(u);
                issue_window(u, 0, stall ? 16u : 0u);
                h_cur = h_next;
                if (u + stride < units) fetch(u + stride);
            }
            auto store_readout = [&](long long uu, int2 hr) {
                if (hr.x > 0) {
                    const long long row0 = (uu / p.H) * p.R + hr.y;
                    bulk_s2g(static_cast<unsigned char*>(p.sketch) + row0 * TV * esz, sm + L.ust, unsigned(hr.x * TV * esz));
                }
                if (p.has_token) bulk_s2g(p.out + uu * TV, sm + L.ust + E * TV * 4, TV * 4);
                bulk_commit();
            };
            unsigned xph = 0;
            for (long long k = 0; u < units; u += stride, ++k) {
                if (!mbar_wait(xbar, xph)) { ok = false; break; }       // the window buffers are free
                xph ^= 1u;
                const int2 h1 = h_next;                                 // head k+1's basis rows
                if (u + stride < units) {
                    issue_window(u + stride, k + 1, 0u);
                    if (u + 2 * stride < units) fetch(u + 2 * stride);
                }
                if (up >= 0) {
                    if (!mbar_wait(rbar, rph)) { ok = false; break; }
                    rph ^= 1u;
                    store_readout(up, h_prev);
                }
                if (!mbar_wait(sbar, sph)) { ok = false; break; }
                sph ^= 1u;
                tph ^= 1u;
                tile_out = false;
                if (n > 0 && up >= 0) {
#pragma unroll
                    for (int bx = 0; bx < TV / 32; ++bx) tma_store_2d(&tmap, 32 * bx, int(up * K), tile + bx * K * 128);
                    bulk_commit();
                }
                bulk_wait_read0();
                mbar_arrive(ebar);                                      // the staging buffers are free
                if (u + stride < units) {
                    issue_state_tile<K, TV>(&tmap, u + stride, tile, tbar);
                    tile_out = true;
                }
                up = u;
                h_prev = h_cur;
                h_cur = h1;
            }
            if (ok && up >= 0) {                                        // the last head's read-out and S_W
                if (mbar_wait(rbar, rph)) {
                    store_readout(up, h_prev);
                    if (n > 0 && mbar_wait(sbar, sph)) {
#pragma unroll
                        for (int bx = 0; bx < TV / 32; ++bx) tma_store_2d(&tmap, 32 * bx, int(up * K), tile + bx * K * 128);
                        bulk_commit();
                    }
                }
            }
            // own copies: one more bounded wait each
            if (tile_out) mbar_wait(tbar, tph);
            if (nwin > 0) mbar_wait(wbar, unsigned((nwin - 1) & 1));
            bulk_wait0();                                               // every store complete
        }
        u = units;                                                      // the loop below is not the mover's
    }

    if (ctl) {
        // ---- the issuing thread: MMA groups as the workers' operands become ready ------------------
        if (issuer) {
            unsigned o1 = 0, o2 = 0, o5 = 0;
            for (int k = 0; u < units; u += stride, ++k) {
                unsigned char* const kub = sm + L.ku[0] + (k & 1) * (NJ * K * 4);
                unsigned char* const kub2 = sm + L.ku2[0] + (k & 1) * (FAM == KDA ? NJ * K * 4 : 0);
                // (1) keys and probes in shared memory, the slow-path verdict set
                if (!mbar_wait(obar1, o1)) { ok = false; break; }
                o1 ^= 1u;
                tc::fence_after();
                const int ne = tab.hr[k & 1] + p.has_token;             // read-out columns
                const bool slow = FAM == KDA && *slow_flag != 0;
                if (!slow) mbar_arrive(xbar);                           // the window buffers are free
                // the previous head's MMAs have finished reading W~ and the B buffers
                if (k > 0 && n > 0) {
                    if (!mbar_wait(ubar, uph)) { ok = false; break; }
                    uph ^= 1u;
                }
                tc::fence_after();
                // Gm = [keys | probes] K'^T.  GDN: bf16 operands, the keys exact and
                // the probes in three parts, K = 16 an instruction
                if (FAM == GDN && n > 0) {
                    const uint32_t id_g = tc::idesc_bf16(128, NJ);
                    const uint32_t s_g16 = smem_u32(sm + L.g16), s_k16 = smem_u32(sm + L.k16);
#pragma unroll 1
                    for (int q = 0; q < K / 16; ++q) {
                        const uint32_t ko = (q & 3) * 32;
                        const uint64_t a = tc::sdesc(s_g16 + (q >> 2) * (128 * 128) + ko, 16, 1024, tc::LAYOUT_SW128);
                        const uint64_t bk = tc::sdesc(s_k16 + (q >> 2) * (NJ * 128) + ko, 16, 1024, tc::LAYOUT_SW128);
                        tc::mma_ss_bf16(tmem + T_W, a, bk, id_g, q > 0);
                    }
                } else if (!slow && n > 0) {
                    const uint32_t id_g = tc::idesc_tf32(128, NG, 0, 0);
                    const uint32_t s_b = FAM == KDA ? s_kq : s_bp;
                    const int brows = FAM == KDA ? 2 * NJ : NB;
#pragma unroll 1
                    for (int q = 0; q < K / 8; ++q) {
                        const uint32_t ko = (q & 3) * 32;
                        const uint64_t a = tc::sdesc(s_bp + (q >> 2) * (NB * 128) + ko, 16, 1024, tc::LAYOUT_SW128);
                        const uint64_t bk = tc::sdesc(s_b + (q >> 2) * (brows * 128) + ko, 16, 1024, tc::LAYOUT_SW128);
                        tc::mma_ss(tmem + T_W, a, bk, id_g, q > 0);
                    }
                }
                tc::commit(gbar);
                ++ng;
                // (2) S_0 in TMEM (the previous head's read-out has read the correction)
                if (!mbar_wait(obar2, o2)) { ok = false; break; }
                o2 ^= 1u;
                tc::fence_after();
                // D = S_0^T [keys | probes]: the hi half against every row, the lo half against the first 16 + E
                const uint32_t id_hi = tc::idesc_tf32(TV, NB, 0, 0), id_lo = tc::idesc_tf32(TV, 16 + E, 0, 0);
#pragma unroll 1
                for (int q = 0; q < K / 8; ++q) {
                    const uint64_t bd = tc::sdesc(s_bp + (q >> 2) * (NB * 128) + (q & 3) * 32, 16, 1024, tc::LAYOUT_SW128);
                    tc::mma_ts(tmem + T_D, tmem + T_HI + 8 * q, bd, id_hi, q > 0);
                    tc::mma_ts(tmem + T_D, tmem + T_LO + 8 * q, bd, id_lo, 1);
                }
                tc::commit(pbar);
                ++np;
                // (5) W~ in TMEM and k^.x in shared memory (Gm and the pass were read)
                if (!mbar_wait(obar5, o5)) { ok = false; break; }
                o5 ^= 1u;
                tc::fence_after();
                // Dc = W~^T (K^ X^T) into the first E columns of the S_0 region (read by the
                // next head's workers before its S_0 lands there), then C += W~^T K^; each
                // group completes on its own mbarrier (committed even when empty)
                const int nq = (n + 7) / 8;
                if (n > 0 && ne > 0) {
                    const uint32_t id_x = tc::idesc_tf32(TV, E, 0, 0);
                    for (int q = 0; q < nq; ++q) {
                        const uint64_t xh = tc::sdesc(s_kxh + q * 32, 16, 1024, tc::LAYOUT_SW128);
                        const uint64_t xl = tc::sdesc(s_kxl + q * 32, 16, 1024, tc::LAYOUT_SW128);
                        tc::mma_ts(tmem + T_HI, tmem + T_W + 8 * q, xh, id_x, q > 0);
                        tc::mma_ts(tmem + T_HI, tmem + T_W + 8 * q, xl, id_x, 1);
                        tc::mma_ts(tmem + T_HI, tmem + T_W + 16 + 8 * q, xh, id_x, 1);
                    }
                }
                tc::commit(cbar);
                ++nc;
                if (n > 0) {
                    const uint32_t id_u = tc::idesc_tf32(TV, K, 0, 1);
                    const uint32_t s_ku = smem_u32(kub), s_ku2 = smem_u32(kub2);
                    for (int q = 0; q < nq; ++q) {
                        const uint64_t bh = tc::sdesc(s_ku + q * 1024, NJ * 128, 512, tc::LAYOUT_SW128_32B);
                        tc::mma_ts(tmem + T_C, tmem + T_W + 8 * q, bh, id_u, 1);
                        tc::mma_ts(tmem + T_C, tmem + T_W + 16 + 8 * q, bh, id_u, 1);
                        if (FAM == KDA)
                            tc::mma_ts(tmem + T_C, tmem + T_W + 8 * q,
                                       tc::sdesc(s_ku2 + q * 1024, NJ * 128, 512, tc::LAYOUT_SW128_32B), id_u, 1);
                    }
                    tc::commit(ubar);
                    ++nu;
                }
            }
        }
        u = units;                                                      // the loop below is the workers'
    }

    // ---- the workers ----------------------------------------------------------------------------------
    // the previous head, whose read-out and S_W are finished during this one
    long long u_prev = -1;
    int ne_prev = 0, r_prev = 0;
    float g_prev = 1.f;
    for (int k = 0; u < units; u += stride, ++k) {
        unsigned char* const kub = sm + L.ku[0] + (k & 1) * (NJ * K * 4);            // this head's update keys
        unsigned char* const kub2 = sm + L.ku2[0] + (k & 1) * (FAM == KDA ? NJ * K * 4 : 0);
        bool fail = false, slow = false;
        uint32_t vv[NJ / 2];                                            // this column's values, bf16 pairs
        float g1 = 1.f;                                                 // GDN: A(n-1,-1)
        float rx[16], rtok = 0.f;                                       // the previous head's read-out

        // the window (this barrier also ends every worker's use of the previous
        // head's tables and buffers)
        if (wsync_or(!mbar_wait(wbar, wph))) { ok = false; break; }
        wph ^= 1u;
        const int r_h = tab.hr[k & 1];                                  // written before the window was issued
        const int ne = r_h + p.has_token;                               // read-out columns [Omega_h | q]
        {
            // ---- phase 1x: values, scalars, keys, probes (the window buffers) ----------------------
#pragma unroll
            for (int j = 0; j < NJ / 2; ++j) {
                const uint32_t a = (hk == 0 && 2 * j < n) ? vraw[2 * j * TV + v] : 0u;
                const uint32_t b = (hk == 0 && 2 * j + 1 < n) ? vraw[(2 * j + 1) * TV + v] : 0u;
                vv[j] = a | (b << 16);
            }
            if (t < NJ) {                                               // b_t and the GDN decays
                float a = 1.f, bt = 0.f;
                if (t < n) {
                    const bool tok = t >= p.n_ring;
                    bt = tok ? tab.tok[0] : sb[t];
                    if (FAM == GDN) a = tok ? tab.tok[1] : sg[t];
                }
                tab.al[t] = a;
                tab.cb[t] = bt;
            }
            bool tiny = false;
            if constexpr (FAM == GDN) {
#pragma unroll
                for (int i = t; i < NJ * (K / 4); i += NWK) {
                    const int j = i / (K / 4), c = (i % (K / 4)) * 4;
                    uint2 w = make_uint2(0u, 0u);
                    if (j < n) w = *reinterpret_cast<const uint2*>(kraw + j * K + c);
                    const float4 v4 = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
                    *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, j, c)) = v4;
                    *reinterpret_cast<float4*>(kub + tc::sw32b_off(NJ, j, c)) = v4;
                    // Gm in bf16: the keys as its B operand and as A's first rows
                    *reinterpret_cast<uint2*>(sm + L.k16 + tc::sw128h_off(NJ, j, c)) = w;
                    *reinterpret_cast<uint2*>(sm + L.g16 + tc::sw128h_off(128, j, c)) = w;
                }
            } else if (t < 2 * K) {
                if (t < K) tiny = kda_keys<K, 0>(t, n, E, NB, kraw, graw, bp, sm + L.kq, kub, kub2, tab.gw);
                else tiny = kda_keys<K, 1>(t - K, n, E, NB, kraw, graw, bp, sm + L.kq, kub, kub2, tab.gw);
            }
            // KDA: the previous head's read-out, from TMEM: its correction was
            // issued as this head began and has had phase 1 to complete.  The
            // values wait in registers until the staging buffer is free (after
            // the operands are in).  (GDN, whose phase 1 is shorter, reads it in
            // one piece after the operands.)
            bool cf = false;
            if (FAM == KDA && u_prev >= 0) {
                cf = !mbar_wait(cbar, cph);
                tc::fence_after();
                if (!cf) ro_load(ne_prev, r_prev, g_prev, rx, rtok);
            }
            const bool v1 = wsync_or(tiny || cf);                       // tab.gw is written
            if (v1 && wsync_or(cf)) { ok = false; break; }
            slow = v1 && FAM == KDA;
            // the probes (KDA: scaled by G(n-1,-1)), hi and lo halves; rows past
            // ne keep stale values, which only reach columns no one reads
#pragma unroll 2
            for (int idx = t; idx < ne * (K / 4); idx += NWK) {
                const int e = idx / (K / 4), c = (idx % (K / 4)) * 4;
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < r_h) {
                    x = *reinterpret_cast<const float4*>(braw + e * K + c);
                } else if (e == r_h && p.has_token) {
                    const uint2 w = *reinterpret_cast<const uint2*>(tq + c);
                    x = make_float4(bf2f_lo(w.x), bf2f_hi(w.x), bf2f_lo(w.y), bf2f_hi(w.y));
                }
                if (FAM == KDA) x = mul4(x, *reinterpret_cast<const float4*>(tab.gw + c));
                const float4 hi = hi4(x);
                *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, 16 + e, c)) = hi;
                *reinterpret_cast<float4*>(bp + tc::sw128_off(NB, 16 + E + e, c)) =
                    make_float4(x.x - hi.x, x.y - hi.y, x.z - hi.z, x.w - hi.w);
                if constexpr (FAM == GDN) {
                    // Gm's A rows in bf16: x = p1 + p2 + p3 exactly (each part the
                    // rounded remainder of the previous ones)
                    float4 r = x;
#pragma unroll
                    for (int pi = 0; pi < 3; ++pi) {
                        const uint2 h = bf16x4(r);
                        *reinterpret_cast<uint2*>(sm + L.g16 + tc::sw128h_off(128, 16 + pi * E + e, c)) = h;
                        r = make_float4(r.x - bf2f_lo(h.x), r.y - bf2f_hi(h.x), r.z - bf2f_lo(h.y), r.w - bf2f_hi(h.y));
                    }
                }
            }
            if (FAM == GDN) {                                           // A(n-1,-1), as a product tree
                float g4[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int i = 0; i < NJ; ++i) g4[i & 3] *= i < n ? tab.al[i] : 1.f;
                g1 = (g4[0] * g4[1]) * (g4[2] * g4[3]);
            }
            tc::fence_proxy_async();
        }
        if (t == 0) *slow_flag = slow ? 1 : 0;
        mbar_arrive(obar1);                                             // (1) operands in shared memory

        {
            // the previous head's read-out into the staging buffer for the mover
            bool ef = false;
            if (FAM == KDA && u_prev >= 0) {
                ef = !mbar_wait(ebar, eph);
                eph ^= 1u;
                if (!ef) ro_stage(ne_prev, r_prev, rx, rtok);
            } else if (u_prev >= 0) {
                ef = readout(ne_prev, r_prev, g_prev);
            }
            // the tile (earlier barriers ordered the TMEM Dc reads before S_0 lands there)
            fail = wsync_or(ef || !mbar_wait(tbar, tph));
            // ---- phase 1y: S_0 into TMEM (beside Gm) ---------------------------------------------------
            if (!fail) {
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
                tc::wait_st();
            }
        }
        if (fail) { ok = false; break; }
        tph ^= 1u;
        if (u_prev >= 0) cph ^= 1u;
        tc::fence_before();
        mbar_arrive(obar2);                                             // (2) S_0 in TMEM, tile read

        {
            // ---- phase 2 (beside the pass) -----------------------------------------------------------
            if (n > 0) {
                // the previous head's S_W (in C) to the tile buffer, then C = Diag(g) S_0
                if (u_prev >= 0) fail = stage_sw();
                else mbar_arrive(sbar);                                 // the tile is read
                if (!fail) {
#pragma unroll 1
                    for (int k0 = 0; k0 < KH; k0 += 32) {
                        const int kb = hk * KH + k0;
                        uint32_t sh[2][16];
                        tc::ld16(tmem + lane_q + T_HI + kb, sh[0]);
                        tc::ld16(tmem + lane_q + T_HI + kb + 16, sh[1]);
                        tc::wait_ld();
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
                // Gm's pieces to shared memory: row r of the pass buffer is TMEM lane r,
                // read by the workers of the first half (one lane quarter per warp)
                if (!fail) fail = wsync_or(!mbar_wait(gbar, gph));
                tc::fence_after();
                if (!fail && !slow && hk == 0) {
                    const int r = v;                                    // TMEM lane = B-buffer row
                    uint32_t g0[16], g1r[16];
                    tc::ld16(tmem + lane_q + T_W, g0);
                    if (FAM == KDA) tc::ld16(tmem + lane_q + T_W + 16, g1r);
                    tc::wait_ld();
                    float* dst = nullptr;
                    bool both = FAM == KDA;                             // add the K' lo columns
                    if (r < 16) dst = pa + r * NJ;
                    else if (r < 16 + E) dst = xa + (r - 16) * NJ;
                    else if (r < 16 + 2 * E) { dst = xb + (r - 16 - E) * NJ; both = false; }
                    else if (FAM == KDA && r < 32 + 2 * E) { dst = pb + (r - 16 - 2 * E) * NJ; both = false; }
                    else if (FAM == GDN && r < 16 + 3 * E) dst = xc + (r - 16 - 2 * E) * NJ;
                    if (dst != nullptr) {
#pragma unroll
                        for (int j = 0; j < NJ; ++j)
                            dst[j] = __uint_as_float(g0[j]) + (both ? __uint_as_float(g1r[j]) : 0.f);
                    }
                }
                if (FAM == KDA && slow && !fail) {
                    // channel by channel: pair weights with the ratio G(t,j)[c] as a
                    // running product (thread (j = t / 16, group cg = t % 16)), and
                    // k^_j . x_e from the update keys and the unscaled probes
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
                    if (cg == 0) {
#pragma unroll
                        for (int q = 0; q < NJ; ++q) {
                            pa[q * NJ + j] = acc[q];
                            pb[q * NJ + j] = 0.f;
                        }
                    }
                    for (int idx = t; idx < E * NJ; idx += NWK) {
                        const int e = idx / NJ, jj = idx % NJ;
                        float s = 0.f;
                        if (jj < n && e < ne) {
                            for (int c = 0; c < K; ++c) {
                                const uint32_t o = tc::sw32b_off(NJ, jj, c);
                                const float kk = *reinterpret_cast<const float*>(kub + o) +
                                                 *reinterpret_cast<const float*>(kub2 + o);
                                const float x = e < r_h ? braw[e * K + c] : bf2f(tq[c]);
                                s = fmaf(kk, x, s);
                            }
                        }
                        xa[idx] = s;
                        xb[idx] = 0.f;
                    }
                }
            } else {
                mbar_arrive(sbar);                                      // the tile is read
            }
            wsync();                                                    // (3) Gm's pieces
            if (t == 0 && slow) mbar_arrive(xbar);                      // KDA slow path: the window buffers are free now
            // k^_j . x_e as the correction's B operand (K-major [e][j]), hi and lo
            for (int idx = t; idx < E * NJ; idx += NWK) {
                const int e = idx / NJ, j = idx % NJ;
                const float x = (j < n && e < ne) ? xa[idx] + xb[idx] + (FAM == GDN ? xc[idx] : 0.f) : 0.f;
                const float hi = tf32_hi(x);
                *reinterpret_cast<float*>(sm + L.kxh + tc::sw128_off(E, e, j)) = hi;
                *reinterpret_cast<float*>(sm + L.kxl + tc::sw128_off(E, e, j)) = x - hi;
            }
            tc::fence_proxy_async();
            if (t < NJ) {
                const int tt = t;
                float al[NJ], pr[NJ];
#pragma unroll
                for (int i = 0; i < NJ; ++i) {
                    al[i] = tab.al[i];
                    pr[i] = pa[tt * NJ + i] + (FAM == KDA ? pb[tt * NJ + i] : 0.f);
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
#pragma unroll
                for (int j = 0; j < NJ; ++j) tab.P[tt * NJ + j] = (j < tt && tt < n) ? pr[j] : 0.f;
            }
            wsync();                                                    // (4) tables

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
                    const float vt = (tt & 1) ? bf2f_hi(vv[tt >> 1]) : bf2f_lo(vv[tt >> 1]);
                    float x = tab.cb[tt] * vt - tab.cy[tt] * y[tt];
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
                tc::st16(tmem + lane_q + T_W, wh);
                tc::st16(tmem + lane_q + T_W + 16, wl);
                tc::wait_st();
            }
        }
        if (fail) { ok = false; break; }
        gph ^= 1u;
        pph ^= 1u;
        if (u_prev >= 0 && n > 0) uph ^= 1u;                            // the previous update, waited in phase 2
        tc::fence_before();
        mbar_arrive(obar5);                                             // (5) W~ and k^.x ready
        u_prev = u;
        ne_prev = ne;
        r_prev = r_h;
        g_prev = FAM == GDN ? g1 : 1.f;
    }
    // the last head's read-out and S_W (staged by the workers, stored by the mover)
    if (!ctl && !mov && ok && u_prev >= 0) {
        bool f = readout(ne_prev, r_prev, g_prev);
        if (!f && n > 0) f = stage_sw();
        if (f) ok = false;
    }
    // a bounded wait ran out: report it; the issuer waits (bounded) for its last
    // MMA groups before the tensor memory is released
    if (!ok && (issuer || mover || t == 0)) report_timeout(p.status);
    if (issuer) {
        if (ng > 0) mbar_wait(gbar, (ng - 1) & 1u);
        if (np > 0) mbar_wait(pbar, (np - 1) & 1u);
        if (nc > 0) mbar_wait(cbar, (nc - 1) & 1u);
        if (nu > 0) mbar_wait(ubar, (nu - 1) & 1u);
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
