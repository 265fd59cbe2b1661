"""Plain fp64 CPU oracle of the SketchSSM decode path.

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA library.  It
may be imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``; the library
(``ssm_decode_b200``) never imports it, and it imports nothing from the
library.  Everything is float64, serial, unblocked and unfused; the only
vectorisation is over independent (sequence, head) pairs and the only library
primitives are numpy element-wise ops, sums and small matrix products.

What it computes, and where each step is defined (page titles and sections):

* Recurrent state update ``S_t = M_t S_{t-1} + B_t`` -- SketchSSM project
  page, "01 / The idea", equation "Full state".  The state is dk x dv and is
  read as ``o_t = S_t^T q_t`` (project page, "02 / How to Make a Sketch": the
  transpose S0^T is V x K and the sketch column is u_i = S0^T omega_i).  The
  pages do not print the three families' M_t and B_t; this oracle takes the
  published forms (reading P1 below).
* Effective query ``q~`` (the query mapped back through the window's buffered
  transitions) and the exact contribution of the buffered updates -- paper
  §3.2 and §C.1 (paperlayer summary of arXiv 2609.33051v2); project page,
  "Between flushes · Non-flush": the buffered updates' own output is added
  exactly.
* Sketch ``U = S0^T Omega`` -- project page, "02 / How to Make a Sketch",
  "Precompute the basis outputs" (u_i = S0^T omega_i).
* Coefficients and readout ``c_t = C q~_t``, ``o^_t = U c_t`` -- project page,
  "Per step · Non-flush: Coefficient vector & readout".
* Flush: apply the W buffered updates to the full state, emit the exact
  output from the updated state, refresh the sketch -- paper §4.1 and App. B
  (paperlayer summary); GitHub repository page, "Overview".
* Schedule: W-1 non-flush steps then one flush per window -- paper App. B.

Readings of points the pages leave open:

* P1 family transitions (B_t = b_t k_t v_t^T in all three):
    Mamba-2: M_t = a_t I, a_t = exp(dt_t A_h), b_t = dt_t  (no erase term,
             consistent with "q~ = d[t] ⊙ q_t" in §C.1);
    GDN:     M_t = a_t (I - beta_t k_t k_t^T), b_t = beta_t;
    KDA:     M_t = (I - beta_t k_t k_t^T) Diag(a_t), a_t in (0,1)^dk, b_t = beta_t.
* P2 update-then-read: ``o_t = S_t^T q_t`` (the flush computes its output
  from the updated state, App. B).
* P4 the coefficient map is either a fixed per-head matrix C (the workloads
  use C = P^T) or the state-dependent map of the project page ("Per window ·
  Flush: Sketch & coefficient map", C = (U^T U)^+ U^T S0^T; paper §A.2.1),
  refreshed with the sketch at every flush.  The pages compare against an
  exact map with a regulariser whose value they do not give; this oracle takes a ridge
  relative to the Gram matrix's mean diagonal, lambda = rho * tr(U^T U) / r,
  so that rho = 0 is the pseudoinverse form for a full-column-rank U.  With a
  bf16 sketch the map is built from the stored (rounded) U and is itself
  stored rounded to bf16 (App. D has non-flush steps read both in BF16).
  The pages' cheaper variant (§A.2.2: the state metric approximated as low
  rank plus diagonal with P = 4 pivots) is read as keeping the n_piv output
  columns of S with the most energy exactly and the rest as a diagonal
  (coefficient_map_lrd); a session can refresh that map instead
  (``map_kind="lrd"``).
* P7 a bf16 sketch is the fp64 sketch rounded once to bf16 (nearest, ties
  to even).

Pins that tie these functions to something other than themselves live in
``tests/test_oracle_pins.py`` (closed forms, brute force over exact
rationals in ``oracle/bruteforce.py``, invariants stated on the pages, and the
delta rule's write/read property).
"""
from __future__ import annotations

import numpy as np

MAMBA2, GDN, KDA = 0, 1, 2


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even).

    bf16 keeps 8 significant bits and fp32's exponent range: the spacing of
    representable values in [2^e, 2^(e+1)) is 2^(e-7), never finer than the
    subnormal spacing 2^-133.  Values past the largest finite bf16 become inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    _, e = np.frexp(x[nz])                    # |x| in [2^(e-1), 2^e)
    step = np.ldexp(1.0, np.maximum(e - 8, -133))
    out[nz] = np.rint(x[nz] / step) * step    # np.rint: half to even
    big = np.abs(out) > 3.3895313892515355e38
    out[big] = np.copysign(np.inf, out[big])
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


# ----------------------------------------------------------------------------
# one token's transition
# ----------------------------------------------------------------------------
def transition_params(family: int, gate, beta, A=None):
    """(a_t, b_t) of one token for every (sequence, head).

    gate/beta are the raw per-token inputs: Mamba-2 gate = dt (beta unused),
    GDN gate = a (scalar), KDA gate = a (vector over dk).  A is the per-head
    Mamba-2 decay rate, broadcastable against dt.
    """
    gate = np.asarray(gate, dtype=np.float64)
    if family == MAMBA2:
        dt = gate
        return np.exp(dt * np.asarray(A, dtype=np.float64)), dt
    return gate, np.asarray(beta, dtype=np.float64)


def apply_transition(family: int, S, k, a, b):
    """M_t S for a batch of dk x dv states S[..., K, V]."""
    if family == MAMBA2:
        return a[..., None, None] * S
    if family == GDN:
        ktS = np.einsum("...k,...kv->...v", k, S)
        return a[..., None, None] * (S - b[..., None, None] * k[..., :, None] * ktS[..., None, :])
    if family == KDA:
        T = a[..., :, None] * S                      # Diag(a_t) S
        ktT = np.einsum("...k,...kv->...v", k, T)
        return T - b[..., None, None] * k[..., :, None] * ktT[..., None, :]
    raise ValueError(family)


def apply_transition_T(family: int, x, k, a, b):
    """M_t^T x for a batch of dk-vectors x[..., K]."""
    if family == MAMBA2:
        return a[..., None] * x
    kx = np.einsum("...k,...k->...", k, x)
    erased = x - (b * kx)[..., None] * k              # (I - b k k^T) x  (symmetric)
    if family == GDN:
        return a[..., None] * erased
    if family == KDA:
        return a * erased                             # Diag(a) (I - b k k^T) x
    raise ValueError(family)


def update(family: int, S, k, v, a, b):
    """S_t = M_t S_{t-1} + b_t k_t v_t^T  (project page, "Full state")."""
    return apply_transition(family, S, k, a, b) + b[..., None, None] * k[..., :, None] * v[..., None, :]


def read(S, q):
    """o = S^T q for states S[..., K, V] and queries q[..., K]."""
    return np.einsum("...kv,...k->...v", S, q)


# ----------------------------------------------------------------------------
# windowed form
# ----------------------------------------------------------------------------
def effective_query(family: int, tokens, q):
    """Effective query and the buffered updates' exact output term.

    ``tokens`` is the window's buffered updates in arrival order, each a tuple
    (k, v, a, b); the query q belongs to the last of them.  With x_tau = q and
    x_{j-1} = M_j^T x_j, the effective query is q~ = x_0 and the buffered
    term is sum_j B_j^T x_j = sum_j b_j (k_j . x_j) v_j, so that
    S_tau^T q = S0^T q~ + o_buf for S_tau the state after the tau updates.
    """
    if not tokens:
        raise ValueError("a window read always includes the query's own update")
    x = np.array(q, dtype=np.float64, copy=True)
    o_buf = None
    for (k, v, a, b) in reversed(tokens):
        kx = np.einsum("...k,...k->...", k, x)
        term = (b * kx)[..., None] * v
        o_buf = term if o_buf is None else o_buf + term
        x = apply_transition_T(family, x, k, a, b)
    return x, o_buf


def windowed_exact_output(family: int, S0, tokens, q):
    """o = S0^T q~ + o_buf: the exact read of the un-flushed window (paper §3.2)."""
    qt, o_buf = effective_query(family, tokens, q)
    return read(S0, qt) + o_buf


def sketch(S, P):
    """U = S^T P: S [..., K, V], basis P [K, r] -> U [..., V, r] (u_i = S^T omega_i)."""
    return np.einsum("...kv,kr->...vr", S, P)


def sketched_output(U, C, q_tilde, o_buf):
    """o^ = U (C q~) + o_buf (project page, "Coefficient vector & readout").
    C is [r, K] (fixed, shared by the batch) or [..., r, K] (state-dependent)."""
    c = np.einsum("...rk,...k->...r", C, q_tilde)
    return np.einsum("...vr,...r->...v", U, c) + o_buf


def coefficient_map_lrd(S, P, n_piv=4, rho=0.0):
    """The cheaper map of paper §A.2.2 under this reading: the state metric
    H = S S^T (the exact map is C = (P^T H P)^-1 P^T H, since U = S^T P) is
    replaced by H^ = L L^T + D, where L holds the n_piv output columns of S
    with the largest energy ||S[:, v]||^2 (their correlations kept exactly)
    and D = diag of the remaining columns' contribution (their coordinate-wise
    energy).  C = (P^T H^ P + lambda I)^-1 P^T H^, lambda = rho tr(P^T H^ P) / r.
    S [..., K, V], basis P [K, r] -> C [..., r, K]."""
    S = np.asarray(S, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    K, V = S.shape[-2], S.shape[-1]
    r = P.shape[-1]
    if r == 0:
        return np.zeros(S.shape[:-2] + (0, K))
    energy = np.einsum("...kv,...kv->...v", S, S)                      # ||S[:, v]||^2
    order = np.argsort(-energy, axis=-1, kind="stable")
    piv = order[..., :n_piv]
    rest = order[..., n_piv:]
    L = np.take_along_axis(S, piv[..., None, :], axis=-1)               # [..., K, n_piv]
    Sr = np.take_along_axis(S, rest[..., None, :], axis=-1)
    d = np.einsum("...kv,...kv->...k", Sr, Sr)                          # diag of the rest
    H = np.einsum("...kp,...jp->...kj", L, L) + d[..., :, None] * np.eye(K)
    Z = np.einsum("kr,...kj->...rj", P, H)                              # P^T H^
    G = np.einsum("...rj,js->...rs", Z, P)                              # P^T H^ P
    lam = rho * np.trace(G, axis1=-2, axis2=-1) / r
    A = G + lam[..., None, None] * np.eye(r)
    C = np.zeros(Z.shape)
    for idx in np.ndindex(A.shape[:-2]):
        try:
            np.linalg.cholesky(A[idx])
        except np.linalg.LinAlgError:
            continue
        C[idx] = np.linalg.solve(A[idx], Z[idx])
    return C


def coefficient_map(U, S, rho=0.0):
    """State-dependent coefficient map C = (U^T U + lambda I)^{-1} U^T S^T
    (project page, "Per window · Flush: Sketch & coefficient map"; paper
    §A.2.1): the map whose c = C q~ minimises ||S^T q~ - U c||_2 (plus
    lambda ||c||^2).  lambda = rho * tr(U^T U) / r.
    U [..., V, r], S [..., K, V] -> C [..., r, K]."""
    U = np.asarray(U, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    r = U.shape[-1]
    if r == 0:
        return np.zeros(U.shape[:-2] + (0, S.shape[-2]))
    G = np.einsum("...vr,...vs->...rs", U, U)              # U^T U
    Z = np.einsum("...vr,...kv->...rk", U, S)              # U^T S^T
    lam = rho * np.trace(G, axis1=-2, axis2=-1) / r
    A = G + lam[..., None, None] * np.eye(r)
    # A Gram matrix that is not positive definite (e.g. an all-zero state
    # with rho = 0) has no such map; the library then stores zeros.
    C = np.zeros(Z.shape)
    for idx in np.ndindex(A.shape[:-2]):
        try:
            np.linalg.cholesky(A[idx])
        except np.linalg.LinAlgError:
            continue
        C[idx] = np.linalg.solve(A[idx], Z[idx])
    return C


def flush(family: int, S0, tokens, q=None):
    """Apply the buffered updates in order; return (S_W, o_W or None)."""
    S = np.array(S0, dtype=np.float64, copy=True)
    for (k, v, a, b) in tokens:
        S = update(family, S, k, v, a, b)
    return S, (read(S, q) if q is not None else None)


# ----------------------------------------------------------------------------
# a decode session: the schedule of paper App. B over [B][H] heads
# ----------------------------------------------------------------------------
class Session:
    """State of one layer's decode for a batch, advanced one token at a time.

    S is the state at the last flush (for the Standard mode: the current
    state); ring holds this window's buffered tokens; U is the sketch of S
    per head (list over heads of [B, V, r_h]).  Step t (1-based) buffers its
    token at slot (t-1) mod W; steps with t mod W == 0 flush.
    """

    def __init__(self, family, state, window, A=None, basis=None, coef=None,
                 offsets=None, sketch_bf16=False, state_map=False, rho=0.0, dense=None, map_kind="exact"):
        self.family = family
        self.S = np.asarray(state, dtype=np.float64).copy()     # [B, H, K, V]
        self.B, self.H, self.K, self.V = self.S.shape
        self.W = window
        self.A = None if A is None else np.asarray(A, dtype=np.float64)
        self.offsets = None if offsets is None else np.asarray(offsets)
        self.P = self.C = None
        if basis is not None:
            basis = np.asarray(basis, dtype=np.float64)
            coef = np.asarray(coef, dtype=np.float64)
            self.P = [basis[self.offsets[h]:self.offsets[h + 1]].T for h in range(self.H)]
            self.C = [coef[self.offsets[h]:self.offsets[h + 1]] for h in range(self.H)]
        # Dense-fallback heads (paper App. D: they read a BF16 copy of their state):
        # the sketch of P = I is that copy (u_k = S0^T e_k = row k of S0), and
        # the read is S0^T q~ through the identity map.
        self.dense = np.zeros(self.H, bool) if dense is None else np.asarray(dense, bool)
        for h in np.flatnonzero(self.dense):
            self.P[h] = np.eye(self.K)
            self.C[h] = np.eye(self.K)
        self.sketch_bf16 = sketch_bf16
        self.state_map, self.rho = state_map, rho
        self.map_kind = map_kind   # "exact" (§A.2.1) or "lrd" (§A.2.2, coefficient_map_lrd)
        self.ring = []
        self.U = None
        self.Cs = None             # state-dependent maps, list over heads of [B, r_h, K]

    # -- inputs -------------------------------------------------------------
    def token(self, inp):
        """Widen one step's raw inputs; return (q, (k, v, a, b))."""
        q = widen_bf16(inp["q"])
        k = widen_bf16(inp["k"])
        v = widen_bf16(inp["v"])
        A = None if self.A is None else self.A[None, :]
        a, b = transition_params(self.family, inp["gate"], inp["beta"], A)
        return q, (k, v, a, b)

    @property
    def phase(self):
        return len(self.ring)

    # -- sketch ---------------------------------------------------------------
    def _make_sketch(self):
        U = [sketch(self.S[:, h], self.P[h]) for h in range(self.H)]
        if self.sketch_bf16:
            U = [round_bf16(u) for u in U]
        self.U = U
        if self.state_map:
            if self.map_kind == "lrd":
                Cs = [None if self.dense[h] else coefficient_map_lrd(self.S[:, h], self.P[h], 4, self.rho)
                      for h in range(self.H)]
            else:
                Cs = [None if self.dense[h] else coefficient_map(U[h], self.S[:, h], self.rho)
                      for h in range(self.H)]
            self.Cs = [c if c is None or not self.sketch_bf16 else round_bf16(c) for c in Cs]

    def coef(self, h):
        """The coefficient map head h's reads use: [r, K] or [B, r, K]."""
        return self.Cs[h] if self.state_map and not self.dense[h] else self.C[h]

    def packed_map(self):
        """State-dependent maps in the library's packed layout [B][R][K]
        (a dense head's rows, which the library never writes, as zeros)."""
        return np.concatenate([np.zeros((self.B, self.K, self.K)) if c is None else c for c in self.Cs], axis=1)

    def packed_sketch(self):
        """Sketch in the library's packed layout [B][R][V] (row = u_i)."""
        return np.concatenate([np.transpose(u, (0, 2, 1)) for u in self.U], axis=1)

    def prime(self):
        """U = S^T P with nothing buffered (a flush of zero updates)."""
        assert self.phase == 0
        self._make_sketch()

    # -- SketchSSM ------------------------------------------------------------
    def decode(self, inp):
        """Non-flush step: buffer the token, return (sketched o^, exact o)."""
        assert self.phase <= self.W - 2 and self.U is not None
        q, tok = self.token(inp)
        self.ring.append(tok)
        qt, o_buf = effective_query(self.family, self.ring, q)
        self.last_q_tilde, self.last_o_buf = qt, o_buf
        o_hat = np.empty((self.B, self.H, self.V))
        self.last_coefficients = []
        for h in range(self.H):
            C = self.coef(h)
            o_hat[:, h] = sketched_output(self.U[h], C, qt[:, h], o_buf[:, h])
            self.last_coefficients.append(np.einsum("brk,bk->br" if C.ndim == 3 else "rk,bk->br",
                                                    C, qt[:, h]))
        return o_hat, read(self.S, qt) + o_buf

    def flush(self, inp=None, with_sketch=True):
        """Flush step: apply every buffered update (plus this step's token)."""
        q = None
        if inp is not None:
            assert self.phase == self.W - 1
            q, tok = self.token(inp)
            self.ring.append(tok)
        self.S, o = flush(self.family, self.S, self.ring, q)
        self.ring = []
        if with_sketch:
            self._make_sketch()
        else:
            self.U = self.Cs = None
        return o

    def step(self, inp):
        """One SketchSSM decode step following the window schedule."""
        if self.phase == self.W - 1:
            return self.flush(inp), None
        return self.decode(inp)

    # -- baselines --------------------------------------------------------------
    def exact_step(self, inp):
        """Standard: update the full state and read it, every step."""
        assert self.phase == 0
        q, (k, v, a, b) = self.token(inp)
        self.S = update(self.family, self.S, k, v, a, b)
        self.U = None
        return read(self.S, q)

    def replay_step(self, inp):
        """ReplaySSM non-flush step: buffer the token, read the full S0 exactly."""
        assert self.phase <= self.W - 2
        q, tok = self.token(inp)
        self.ring.append(tok)
        return windowed_exact_output(self.family, self.S, self.ring, q)
