// Internal interface between the host API (ss_api.cu) and the kernels
// (ss_kernels.cu).  Not part of the public ABI.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sketchssm.h"

namespace ss {

// Parameters of the state-streaming kernel.  One launch serves ss_prime,
// ss_flush (with or without a token), the ReplaySSM flush and ss_exact_step:
// it applies `n_ring` buffered updates from the ring and, if `has_token`, the
// step's own token as one more update; then it writes the state, the output
// S^T q (if has_token) and the sketch S^T Omega (if do_sketch).
struct FlushParams {
    float* state;
    const uint16_t* ring_k;
    const uint16_t* ring_v;
    const float* ring_gate;
    const float* ring_beta;
    const uint16_t* tok_q;
    const uint16_t* tok_k;
    const uint16_t* tok_v;
    const float* tok_gate;
    const float* tok_beta;
    void* sketch;
    const float* basis;
    const float* A;
    float* out;
    int32_t* status;
    int B, H, W, Wg, R;
    int n_ring, has_token, do_sketch, sketch_bf16;
    int stall;               // testing hook: extra bytes expected by the first bulk wait
    // Mixed-phase steps (ss_step_mixed): only sequences b with fill_in[b] ==
    // W-1 flush; each writes fill_out[b] = 0.  Null for a uniform batch.
    const int32_t* fill_in;
    int32_t* fill_out;
    // State-dependent coefficient map (SS_COEF_STATE): when set, the flush
    // also writes C = (U^T U + lambda I)^-1 U^T S^T, lambda = ridge tr(U^T U)/r,
    // for every head it sketches, as [B][R][dk] in the sketch dtype.
    void* cmap;
    float ridge;
    // SS_COEF_LRD: the map of the low-rank-plus-diagonal state metric instead,
    // C = (P^T H P + lambda I)^-1 P^T H with H = L L^T + D (see build_map).
    int lrd;
    // Dense-fallback heads (bit h): the sketch rows of head h hold a copy of
    // its state, row k = S[k][:], in the sketch dtype, written by the flush
    // instead of S^T Omega; no basis rows are read for them.
    uint32_t dense[SS_MAX_HEADS / 32];
    int off[SS_MAX_HEADS + 1];
};

// Parameters of the ring-append + windowed-read kernels (ss_decode_step and
// ss_replay_step).  The token is appended at ring slot `p`; slots 0..p-1 are
// the window's earlier updates.
struct StepParams {
    const float* state;      // replay only
    uint16_t* ring_k;
    uint16_t* ring_v;
    float* ring_gate;
    float* ring_beta;
    const uint16_t* tok_q;
    const uint16_t* tok_k;
    const uint16_t* tok_v;
    const float* tok_gate;
    const float* tok_beta;
    const void* sketch;      // decode only
    const float* coef;       // decode only
    const float* A;
    float* out;
    int32_t* status;
    int B, H, W, Wg, R;
    int p, sketch_bf16;
    int stall;               // testing hook: extra bytes expected by the first bulk wait
    // Mixed-phase steps (ss_step_mixed): sequence b appends at slot fill_in[b]
    // (p is then the largest slot, W-2, which sizes the staging); sequences
    // with fill_in[b] == W-1 are left to the flush; each other sequence
    // writes fill_out[b] = fill_in[b] + 1.  Null for a uniform batch.
    const int32_t* fill_in;
    int32_t* fill_out;
    // SS_COEF_STATE: per-unit maps [B][R][dk] in the sketch dtype, staged with
    // each unit instead of the shared `coef` (decode only).
    const void* cmap;
    // Dense-fallback heads (bit h): the read is S0^T q~ from the state copy in
    // the sketch rows, streamed from HBM; no map, nothing staged for it.
    // dense_any: some head is dense (the unit buffer then holds q~, dk floats).
    uint32_t dense[SS_MAX_HEADS / 32];
    int dense_any;
    int off[SS_MAX_HEADS + 1];
};

__host__ __device__ inline bool head_dense(const uint32_t* mask, int h) { return (mask[h >> 5] >> (h & 31)) & 1u; }

// Launchers return the launch's cudaError_t (cudaSuccess when queued).
// `rmax` is the largest per-head rank taking part in the launch.
cudaError_t launch_flush(int family, int dk, int dv, const FlushParams& p, int rmax,
                         cudaStream_t stream);
// Mamba-2 flush on the tensor cores (any dk, dv in {64, 128}).
cudaError_t launch_flush_mma(int dk, int dv, const FlushParams& p, int rmax, cudaStream_t stream);
// GDN / KDA flush on the fifth-generation tensor cores (dv = 128, dk in
// {64, 128}, at most 16 updates and 32 read-out columns, uniform batch, fixed
// coefficient map); flush_tc_eligible tells whether a launch qualifies.
bool flush_tc_eligible(int family, int dk, int dv, const FlushParams& p, int rmax);
cudaError_t launch_flush_tc(int family, int dk, const FlushParams& p, int rmax, cudaStream_t stream);
// After a flush with a sketch: the dense-fallback heads' state copies.
cudaError_t launch_dense_copy(int dk, int dv, const FlushParams& p, cudaStream_t stream);
int flush_mma_smem_bytes(int dk, int dv, int n, int e16);
cudaError_t launch_decode(int family, int dk, int dv, const StepParams& p, int rmax,
                          cudaStream_t stream);
cudaError_t launch_replay(int family, int dk, int dv, const StepParams& p,
                          cudaStream_t stream);

}  // namespace ss
