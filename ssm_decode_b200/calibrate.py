"""Offline calibration on seeded synthetic samples: sketch bases and ranks.

Host-side preprocessing that runs once per model, never on the decode path
(numpy, fp64).  It produces what the decode library consumes: per-head basis
rows Omega (the `basis` buffer), the matching fixed coefficient map C (the
`coef` buffer) and the per-head ranks / dense-fallback flags of ss_config.

* Basis (SketchSSM project page, "How to Make a Sketch", "Offline · Fixed:
  Sketching matrix"; paper §A.1): with the average state geometry
  E0 = E[S0 S0^T] and z = E0^{1/2} q~, P_G holds the top G eigenvectors of
  E[z z^T] (uncentered PCA) and Omega* = E0^{-1/2} P_G minimises
  L_G(Omega) = E min_c ||E0^{1/2} (q~ - Omega c)||^2.  For that Omega the
  minimising coefficients are c = P_G^T E0^{1/2} q~, so the fixed map is
  C* = P_G^T E0^{1/2} (Omega*^T E0 Omega* = I).
* Ranks (paper §4.2 and App. E): every head has candidate prefix ranks of
  its basis, each with a score (reconstruction error weighted by the head's
  loss sensitivity) and a traffic cost, plus a dense-fallback option (error
  0, the cost of reading a bf16 state copy).  A traffic price lambda makes
  the heads independent (each takes argmin score + lambda * cost); lambda is
  bisected until the total traffic meets the budget; the best feasible
  allocation is kept and the remaining slack is spent on improving
  single-head substitutions.

The pages calibrate on model states and WikiText-2 continuations and pair
the error with output-gradient sensitivity; neither exists here, so the
samples are the synthetic generator's seeded states and queries and the
sensitivity is a seeded positive weight per head (stated by the caller).
"""
from __future__ import annotations

import dataclasses

import numpy as np


# ----------------------------------------------------------------------------
# basis
# ----------------------------------------------------------------------------
def _sym_pow(A, p):
    """A^p for a symmetric positive definite A (eigendecomposition)."""
    w, Q = np.linalg.eigh(A)
    w = np.maximum(w, np.finfo(np.float64).tiny)
    return (Q * w ** p) @ Q.T


@dataclasses.dataclass
class HeadBasis:
    omega: np.ndarray       # [K, G]   Omega* = E0^{-1/2} P_G (columns = basis vectors, by energy)
    coef: np.ndarray        # [G, K]   C*    = P_G^T E0^{1/2}
    energy: np.ndarray      # [K]      eigenvalues of E[z z^T], descending
    E0: np.ndarray          # [K, K]


def fit_head_basis(states, queries, G=None):
    """Omega* for one head from samples.

    states  [N, K, V]: window-boundary states S0 (their average geometry E0);
    queries [M, K]:    effective queries q~ seen against them.
    Returns the basis of every prefix rank at once (columns sorted by captured
    energy), so rank r uses omega[:, :r] and coef[:r]."""
    S = np.asarray(states, dtype=np.float64)
    q = np.asarray(queries, dtype=np.float64)
    K = S.shape[1]
    G = K if G is None else G
    E0 = np.einsum("nkv,njv->kj", S, S) / len(S)
    E0h, E0mh = _sym_pow(E0, 0.5), _sym_pow(E0, -0.5)
    z = q @ E0h.T                                          # z = E0^{1/2} q~
    Czz = z.T @ z / len(z)                                 # uncentered second moment
    w, Q = np.linalg.eigh(Czz)
    order = np.argsort(w)[::-1]
    w, Q = w[order], Q[:, order]
    PG = Q[:, :G]
    return HeadBasis(omega=E0mh @ PG, coef=PG.T @ E0h, energy=w, E0=E0)


def reconstruction_error(hb: HeadBasis, states, queries, r):
    """Mean ||S0^T q~ - U c||^2 with U = S0^T Omega_r, c = C_r q~ over all
    (state, query) pairs: the read error of rank r with the fixed map."""
    S = np.asarray(states, dtype=np.float64)
    q = np.asarray(queries, dtype=np.float64)
    proj = hb.omega[:, :r] @ hb.coef[:r] if r > 0 else np.zeros((S.shape[1],) * 2)
    d = q - q @ proj.T                                     # q~ - Omega C q~
    # E_S ||S^T d||^2 = d^T E0 d
    return float(np.mean(np.einsum("mk,kj,mj->m", d, hb.E0, d)))


def loss_curve(hb: HeadBasis, ranks):
    """Calibration loss L_G at each rank in closed form: the energy of E[z z^T]
    beyond the first r eigenvectors."""
    tail = np.concatenate([np.cumsum(hb.energy[::-1])[::-1], [0.0]])
    return np.array([tail[r] for r in ranks])


# ----------------------------------------------------------------------------
# rank allocation
# ----------------------------------------------------------------------------
DENSE = -1          # the dense-fallback option in an allocation


@dataclasses.dataclass
class Allocation:
    ranks: np.ndarray       # [H] chosen rank, or DENSE
    score: float            # sum of the chosen options' scores
    traffic: float          # sum of their costs


def traffic_per_step(rank, K, V, W, erase=True, dense=False):
    """Non-flush read bytes of one head (paper App. D): bf16 sketch and map,
    G (K + V), plus G W projected erase vectors for GDN/KDA; a dense head reads
    a bf16 K x V state copy."""
    if dense:
        return 2.0 * K * V
    return 2.0 * rank * (K + V) + (2.0 * rank * W if erase else 0.0)


def _choose(scores, costs, lam):
    """Per head, the option minimising score + lam * cost (ties: cheaper)."""
    obj = scores + lam * costs
    best = obj.min(axis=1, keepdims=True)
    # among the options within rounding of the best, take the cheapest
    cand = np.where(obj <= best + 1e-12 * np.maximum(1.0, np.abs(best)), costs, np.inf)
    return np.argmin(cand, axis=1)


def allocate(scores, costs, budget, iters=100):
    """Knapsack allocation by a traffic price, bisection and slack filling.

    scores [H, O], costs [H, O]: each head's options (rows may use +inf for
    options that do not exist).  budget: total cost allowed.  Returns the
    chosen option index per head.  Raises if even the cheapest options do
    not fit."""
    scores = np.asarray(scores, dtype=np.float64)
    costs = np.asarray(costs, dtype=np.float64)
    H = len(scores)
    idx = np.arange(H)
    cheapest = np.argmin(np.where(np.isfinite(scores), costs, np.inf), axis=1)
    if costs[idx, cheapest].sum() > budget:
        raise ValueError("the budget is below the cheapest allocation")
    best = None

    def consider(choice):
        nonlocal best
        t = costs[idx, choice].sum()
        if t <= budget * (1 + 1e-12):
            s = scores[idx, choice].sum()
            if best is None or s < best[0] - 1e-15 or (s <= best[0] + 1e-15 and t < best[1]):
                best = (s, t, choice.copy())

    # bisection on the price: lo gives traffic above the budget, hi below
    lo, hi = 0.0, 1.0
    consider(cheapest)
    if costs[idx, _choose(scores, costs, 0.0)].sum() <= budget:
        consider(_choose(scores, costs, 0.0))
    else:
        while costs[idx, _choose(scores, costs, hi)].sum() > budget:
            hi *= 2.0
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            ch = _choose(scores, costs, mid)
            if costs[idx, ch].sum() > budget:
                lo = mid
            else:
                hi = mid
                consider(ch)
        consider(_choose(scores, costs, hi))
    # slack: the best single-head substitution that still fits, repeatedly
    s, t, choice = best
    while True:
        slack = budget - t
        gain = scores[idx, choice][:, None] - scores               # score saved by switching
        extra = costs - costs[idx, choice][:, None]
        ok = (extra <= slack * (1 + 1e-12)) & (gain > 1e-15) & np.isfinite(scores)
        if not ok.any():
            break
        g = np.where(ok, gain, -np.inf)
        h, o = np.unravel_index(np.argmax(g), g.shape)
        t += extra[h, o]
        s -= gain[h, o]
        choice[h] = o
    return choice


def allocate_ranks(errors, sensitivity, K, V, W, mean_rank, erase=True, max_rank=None, dense=True):
    """Ranks for H heads under the traffic of `mean_rank` on every head.

    errors [H, R+1]: read error of each head at prefix ranks 0..R (R <= K);
    sensitivity [H]: loss weight per head.  Options per head: ranks 1..R and,
    if `dense`, the dense fallback (error 0).  Returns an Allocation with
    ranks[h] in 1..R or DENSE."""
    errors = np.asarray(errors, dtype=np.float64)
    H, R1 = errors.shape
    R = R1 - 1 if max_rank is None else min(max_rank, R1 - 1)
    ranks = np.arange(1, R + 1)
    scores = np.asarray(sensitivity, np.float64)[:, None] * errors[:, 1:R + 1]
    costs = np.broadcast_to([traffic_per_step(r, K, V, W, erase) for r in ranks], scores.shape).copy()
    if dense:
        scores = np.concatenate([scores, np.zeros((H, 1))], axis=1)
        costs = np.concatenate([costs, np.full((H, 1), traffic_per_step(0, K, V, W, erase, dense=True))], axis=1)
    budget = H * traffic_per_step(mean_rank, K, V, W, erase)
    choice = allocate(scores, costs, budget)
    out = np.where(choice < R, ranks[np.minimum(choice, R - 1)], DENSE)
    idx = np.arange(H)
    return Allocation(ranks=out, score=float(scores[idx, choice].sum()), traffic=float(costs[idx, choice].sum()))
