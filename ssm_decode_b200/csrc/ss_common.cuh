// Device helpers shared by the SketchSSM kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "ss_internal.h"

namespace ss {

constexpr int MAMBA2 = SS_MAMBA2, GDN = SS_GDN, KDA = SS_KDA;
constexpr unsigned FULL = 0xffffffffu;
// Running decay products are kept inside [2^-32, 2^32]; outside it the decay is
// folded into the stored state (see flush_kernel).
constexpr float GAMMA_LO = 2.3283064365386963e-10f;
constexpr float GAMMA_HI = 4294967296.0f;
constexpr int SMEM_LIMIT = 227 * 1024;        // dynamic shared memory per CTA
constexpr int SMEM_SM = 228 * 1024;           // shared memory per SM (1 KB of it reserved per CTA)

__host__ __device__ __forceinline__ int align16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ float bf2f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }
__device__ __forceinline__ float bf2f_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf2f_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint16_t f2bf(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Copy `bytes` (a multiple of 16) with `nthreads` cooperating threads.
__device__ __forceinline__ void stage(void* dst, const void* src, int bytes, int t, int nthreads) {
    for (int o = t * 16; o < bytes; o += nthreads * 16)
        cp_async16(static_cast<char*>(dst) + o, static_cast<const char*>(src) + o);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 dup2(float x) { return make_float2(x, x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(FULL, x, m);
    return x;
}

// ---------------------------------------------------------------------------
// Bulk asynchronous copies (TMA, non-tensor) completing on an mbarrier.
// Every wait is bounded by the global nanosecond timer; a wait that runs out
// reports SS_DEVICE_TIMEOUT through the optional status word.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make an mbarrier initialisation visible to the copy engine.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Copy `bytes` (a multiple of 16, both addresses 16-byte aligned) global -> shared.
// Plain arrival (no transaction bytes) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// One bounded probe of an mbarrier phase: the thread may be suspended for up
// to `hint_ns` (woken early when the phase completes), so a waiting warp
// issues few instructions.
#ifndef SS_WAIT_HINT_NS
#define SS_WAIT_HINT_NS 2000
#endif
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned phase) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase), "r"(SS_WAIT_HINT_NS)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}
constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;   // one second

// Wait for the phase `phase` of `bar`; false if the limit ran out first.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, phase))
        if (global_ns() - t0 > WAIT_LIMIT_NS) return false;
    return true;
}

// A mixed step (fill_in set) flushes only the units whose sequence sits at
// the window's last slot, fill_in[b] == W-1.  Each CTA of the flush keeps a
// queue of its own such units in shared memory: its candidates are
// blockIdx.x, blockIdx.x + gridDim.x, ...; warp 0 compacts them 32 at a time
// with a ballot whenever the queue runs dry, so the fill counts are read once
// per candidate and the next unit is a shared-memory read.  The refill also
// writes fill_out[b] = 0 for each flushing sequence (from its head-0 unit).
constexpr int FQ_CAP = 64;
struct FlushQueue {
    long long pos;           // next candidate to test
    long long next;          // the unit handed out last (all threads read it)
    int head, count;         // unit[head..count) are queued
    int unit[FQ_CAP];
};
constexpr int FQ_BYTES = (int(sizeof(FlushQueue)) + 15) & ~15;

__device__ __forceinline__ void fq_init(FlushQueue* q) {          // one thread
    q->pos = blockIdx.x;
    q->next = 0;
    q->head = q->count = 0;
}

// Called by the whole of warp 0: the next unit this CTA flushes (`units`
// when none is left); lane 0 also publishes it in q->next.
__device__ __forceinline__ long long fq_next(const FlushParams& p, FlushQueue* q, long long units) {
    const int lane = threadIdx.x & 31;
    const bool refill = q->head == q->count;
    __syncwarp();                                       // every lane has read head/count
    if (refill) {
        long long pos = q->pos;
        int n = 0;
        while (pos < units && n <= FQ_CAP - 32) {
            const long long c = pos + (long long)lane * gridDim.x;
            const int f = c < units ? p.fill_in[c / p.H] : 0;
            const bool hit = c < units && f == p.W - 1;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (hit) {
                q->unit[n + __popc(m & ((1u << lane) - 1u))] = int(c);
                if (c % p.H == 0) p.fill_out[c / p.H] = 0;   // the sequence's new fill, once per sequence
            } else if (c < units && (f < 0 || f > p.W - 1) && c % p.H == 0 && p.status != nullptr) {
                atomicOr(p.status, SS_DEVICE_BAD_FILL);      // neither flushed nor decoded: reported once
            }
            n += __popc(m);
            pos += 32LL * gridDim.x;
        }
        __syncwarp();
        if (lane == 0) {
            q->pos = pos;
            q->head = 0;
            q->count = n;
        }
        __syncwarp();
    }
    const int h = q->head;
    const long long u = h < q->count ? (long long)q->unit[h] : units;
    __syncwarp();                                       // every lane has read head
    if (lane == 0) {
        if (h < q->count) q->head = h + 1;
        q->next = u;
    }
    __syncwarp();
    return u;
}

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the previous kernel in the stream is still finishing; it runs only
// set-up that touches no global memory (shared memory, mbarriers) before
// griddep_wait(), which returns once the previous kernel has completed and
// its writes are visible, so the data order is the plain stream order.
// griddep_launch_next() then lets the next such kernel start its set-up.
// Both are no-ops for an ordinary launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

__device__ __forceinline__ void report_timeout(int32_t* status) {
    if (status != nullptr) atomicOr(status, SS_DEVICE_TIMEOUT);
}

// Instantiate FN<family, dk, dv> for the runtime (family, dk, dv).
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

// Streaming multiprocessors of the current device (148 on B200), for
// persistent grids.
inline int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

// Host-side cache of one kernel's launch attributes, per device: registers
// per thread (queried once), the dynamic shared-memory limit set so far (the
// attribute is only raised), and the last occupancy answer.  Steady-state
// launches then make no attribute or occupancy queries.
struct KernelCache {
    static constexpr int MAXDEV = 16;
    std::atomic<int> regs[MAXDEV] = {};
    std::atomic<int> smem[MAXDEV] = {};
    std::atomic<long long> occ[MAXDEV] = {};   // (block threads << 40) | (bytes << 8) | blocks per SM
};

inline int cur_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= KernelCache::MAXDEV) d = 0;
    return d;
}

template <typename F>
cudaError_t cached_regs(F kern, KernelCache& kc, int* regs) {
    const int d = cur_device();
    int r = kc.regs[d].load(std::memory_order_relaxed);
    if (r <= 0) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        r = fa.numRegs > 0 ? fa.numRegs : 64;
        kc.regs[d].store(r, std::memory_order_relaxed);
    }
    *regs = r;
    return cudaSuccess;
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes`.  The
// check, the attribute call and the cache update run under one lock, so two
// host threads asking for different sizes cannot leave the attribute below
// the cached value.
inline std::mutex& smem_attr_mutex() {
    static std::mutex mu;
    return mu;
}

template <typename F>
cudaError_t ensure_smem(F kern, KernelCache& kc, int bytes) {
    const int d = cur_device();
    if (bytes <= kc.smem[d].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(smem_attr_mutex());
    if (bytes <= kc.smem[d].load(std::memory_order_relaxed)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) kc.smem[d].store(bytes, std::memory_order_release);
    return e;
}

template <typename F>
cudaError_t cached_occupancy(F kern, KernelCache& kc, int threads, int bytes, int* per_sm) {
    const int d = cur_device();
    const long long key = ((long long)threads << 40) | ((long long)bytes << 8);
    const long long v = kc.occ[d].load(std::memory_order_relaxed);
    if (v != 0 && (v & ~0xffLL) == key) { *per_sm = int(v & 0xff); return cudaSuccess; }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, bytes);
    if (e != cudaSuccess) return e;
    if (n < 1) n = 1;
    if (n > 255) n = 255;
    kc.occ[d].store(key | n, std::memory_order_relaxed);
    *per_sm = n;
    return cudaSuccess;
}

}  // namespace ss
