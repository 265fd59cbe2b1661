"""Seeded synthetic decode workloads for the SketchSSM decode path.

This module only draws random inputs.  It holds none of the method's
arithmetic (no recurrence, no sketch, no readout), so the fp64 oracle and the
CUDA library can both be fed from it without sharing any computation.

Every tensor is produced from numpy's PCG64 with a ``SeedSequence``:
``SeedSequence(1000 * seed_id)`` for the static tensors (initial state, decay
rates, ranks, basis) and ``SeedSequence([1000 * seed_id, step])`` for the
inputs of decode step ``step``, so any step can be regenerated without
storing the stream.

Shapes and distributions follow the workloads on the SketchSSM pages:
window W = 16, mean sketch rank 8, fp32 state, bf16 q/k/v, batch 128..512
(project page, "04 / Linear-attention kernel speedup", Figure 6 caption; paper
§5.2 and §F.1 as summarised on the paperlayer page).  The pages benchmark on
real models; these synthetic tensors stand in for them.

Conventions (N(mean, variance)):
  * state S0 ~ N(0, 0.1), fp32, layout [B][H][dk][dv]
  * Mamba-2: q, k ~ N(0, 1/dk) (or the structured query below), v ~ N(0, 1),
    dt = softplus(N(-2, 1)), A_h = -exp(U(0, 2))
  * GDN: q, k L2-normalised, beta = sigmoid(N(0,1)), a = exp(-softplus(N(0,1)))
  * KDA: as GDN with a per-channel a in (0,1)^dk
  * structured queries: q = G_h z + 0.1 n with G_h = Q_h diag(0.7^i), Q_h a
    Haar-random orthogonal matrix; the basis P_h is Q_h[:, :r_h], i.e. the
    top-r_h eigenvectors of the query covariance G_h G_h^T + 0.01 I.
  * ragged ranks with mean m: uniform on [max(1, m//4), min(2m, dk)], then
    +-1 adjustments until the sum is exactly m * H.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

MAMBA2, GDN, KDA = 0, 1, 2
FAMILY_NAMES = {MAMBA2: "mamba2", GDN: "gdn", KDA: "kda"}


# ----------------------------------------------------------------------------
# bf16 bit patterns (storage format of q/k/v; round-to-nearest-even)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + lsb) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# workload descriptions
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    family: int
    batch: int
    heads: int
    dk: int
    dv: int
    window: int
    steps: int
    mean_rank: int
    seed_id: int
    ragged: bool = True          # ragged per-head ranks (else all = mean_rank)
    structured_q: bool = True    # q = G z + 0.1 n (else isotropic N(0, 1/dk))

    @property
    def units(self) -> int:
        """(sequence, head) pairs per decode step."""
        return self.batch * self.heads


WORKLOADS = {
    # Mamba-2-style scalar decay, the small parity case
    "mamba2_b4": Workload("mamba2_b4", MAMBA2, 4, 4, 64, 64, 16, 64, 8, 1,
                          ragged=False, structured_q=False),
    # Mamba-2 layer decode: batch 320, 128 heads, headdim 64, dstate 128
    "mamba2_b320": Workload("mamba2_b320", MAMBA2, 320, 128, 128, 64, 16, 256, 8, 2),
    # Gated DeltaNet decode: batch 256, 32 heads, dk = dv = 128
    "gdn_b256": Workload("gdn_b256", GDN, 256, 32, 128, 128, 16, 256, 8, 3),
    # KDA decode: batch 256, 32 heads, dk = dv = 128, per-channel decay
    "kda_b256": Workload("kda_b256", KDA, 256, 32, 128, 128, 16, 256, 8, 4),
}

SWEEP_BATCHES = (1, 32, 128, 320, 1024)
SWEEP_WINDOWS = (4, 8, 16, 32)
SWEEP_RANKS = (4, 8, 16)


def sweep_workload(batch: int, window: int, mean_rank: int) -> Workload:
    """One point of the Mamba-2-shape sweep (batch x W x mean rank)."""
    sid = 5000 + 100 * SWEEP_BATCHES.index(batch) + 10 * SWEEP_WINDOWS.index(window) \
        + SWEEP_RANKS.index(mean_rank)
    return Workload(f"mamba2_sweep_b{batch}_w{window}_r{mean_rank}", MAMBA2, batch, 128,
                    128, 64, window, 256, mean_rank, sid)


def shrink(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes replaced (same distributions)."""
    return replace(wl, **kw)


# ----------------------------------------------------------------------------
# static tensors
# ----------------------------------------------------------------------------
def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def draw_ranks(rng: np.random.Generator, heads: int, mean: int, dk: int, ragged: bool) -> np.ndarray:
    if not ragged:
        return np.full(heads, mean, dtype=np.int32)
    lo, hi = max(1, mean // 4), min(2 * mean, dk)
    r = rng.integers(lo, hi + 1, size=heads).astype(np.int64)
    target = mean * heads
    while r.sum() != target:
        if r.sum() > target:
            cand = np.where(r > lo)[0]
            i = cand[np.argmax(r[cand])]
            r[i] -= 1
        else:
            cand = np.where(r < hi)[0]
            i = cand[np.argmin(r[cand])]
            r[i] += 1
    return r.astype(np.int32)


def haar_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


@dataclass
class Static:
    ranks: np.ndarray            # int32 [H]
    offsets: np.ndarray          # int32 [H + 1], packed row offsets into basis / coef / sketch
    state: np.ndarray            # float32 [B][H][dk][dv]
    A: np.ndarray                # float32 [H] (Mamba-2 decay rate, < 0); zeros otherwise
    basis: np.ndarray            # float32 [R][dk]; rows off[h]..off[h]+r_h-1 are head h's omega_i
    coef: np.ndarray             # float32 [R][dk]; head h's coefficient map rows (C = P^T)
    qmix: np.ndarray = field(repr=False, default=None)   # float32 [H][dk][dk]: G_h


def static_inputs(wl: Workload, with_state: bool = True) -> Static:
    rng = _rng(1000 * wl.seed_id)
    ranks = draw_ranks(rng, wl.heads, wl.mean_rank, wl.dk, wl.ragged)
    offsets = np.zeros(wl.heads + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(ranks)
    R = int(offsets[-1])
    basis = np.zeros((R, wl.dk), dtype=np.float32)
    qmix = np.zeros((wl.heads, wl.dk, wl.dk), dtype=np.float32)
    spectrum = 0.7 ** np.arange(wl.dk)
    for h in range(wl.heads):
        Q = haar_orthogonal(rng, wl.dk)
        basis[offsets[h]:offsets[h + 1], :] = Q[:, :ranks[h]].T
        qmix[h] = (Q * spectrum[None, :]).astype(np.float32)
    coef = basis.copy()
    if wl.family == MAMBA2:
        A = (-np.exp(rng.uniform(0.0, 2.0, size=wl.heads))).astype(np.float32)
    else:
        A = np.zeros(wl.heads, dtype=np.float32)
    state = None
    if with_state:
        srng = _rng(1000 * wl.seed_id, 1 << 20)
        state = np.empty((wl.batch, wl.heads, wl.dk, wl.dv), dtype=np.float32)
        for b in range(wl.batch):   # per-sequence draws keep peak memory low
            state[b] = (srng.standard_normal((wl.heads, wl.dk, wl.dv), dtype=np.float32)
                        * np.float32(np.sqrt(0.1)))
    return Static(ranks, offsets, state, A, basis, coef, qmix)


# ----------------------------------------------------------------------------
# per-step inputs
# ----------------------------------------------------------------------------
def _softplus(x):
    return np.logaddexp(0.0, x)


def _l2n(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def step_inputs(wl: Workload, st: Static, step: int) -> dict:
    """Inputs of decode step ``step`` (0-based) for every (sequence, head).

    Returns numpy arrays: q, k [B][H][dk] and v [B][H][dv] as bf16 bits
    (uint16); gate fp32 [B][H] (Mamba-2: dt, GDN: a) or [B][H][dk] (KDA: a);
    beta fp32 [B][H] (zeros for Mamba-2, whose beta is dt).
    """
    rng = _rng(1000 * wl.seed_id, step)
    B, H, K, V = wl.batch, wl.heads, wl.dk, wl.dv
    if wl.structured_q:
        z = rng.standard_normal((H, B, K), dtype=np.float32)
        n = rng.standard_normal((B, H, K), dtype=np.float32)
        q = np.matmul(z, np.transpose(st.qmix, (0, 2, 1))).transpose(1, 0, 2) + 0.1 * n
    else:
        q = rng.standard_normal((B, H, K), dtype=np.float32) / np.sqrt(K)
    k = rng.standard_normal((B, H, K), dtype=np.float32) / np.sqrt(K)
    v = rng.standard_normal((B, H, V), dtype=np.float32)
    if wl.family == MAMBA2:
        gate = _softplus(rng.standard_normal((B, H)) - 2.0).astype(np.float32)
        beta = np.zeros((B, H), dtype=np.float32)
    else:
        q, k = _l2n(q), _l2n(k)
        beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, H))))).astype(np.float32)
        gshape = (B, H) if wl.family == GDN else (B, H, K)
        gate = np.exp(-_softplus(rng.standard_normal(gshape))).astype(np.float32)
    return {
        "q": f32_to_bf16_bits(q.astype(np.float32)),
        "k": f32_to_bf16_bits(k.astype(np.float32)),
        "v": f32_to_bf16_bits(v),
        "gate": np.ascontiguousarray(gate, dtype=np.float32),
        "beta": np.ascontiguousarray(beta, dtype=np.float32),
    }
