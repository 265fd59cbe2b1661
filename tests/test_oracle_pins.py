"""Pins of the fp64 oracle to things other than itself.

Each test ties an oracle function to a closed form, a brute force over exact
rationals, an invariant the SketchSSM pages state, or a defining property of
the delta rule.  ``test_planted_mistakes_are_caught`` plants plausible
mistakes in the oracle (on the CPU) and checks that the pins fail on them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import bruteforce as bf
from oracle import sketchssm_oracle as orc

FAMS = (orc.MAMBA2, orc.GDN, orc.KDA)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers: random fp64 tokens
# ----------------------------------------------------------------------------
def rand_tokens(rng, family, n, K, V, tau, unit_keys=False):
    toks = []
    for _ in range(tau):
        k = rng.standard_normal((n, K))
        if unit_keys or family != orc.MAMBA2:
            k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = rng.standard_normal((n, V))
        if family == orc.MAMBA2:
            a = np.exp(-rng.uniform(0.01, 1.0, n))
            b = rng.uniform(0.05, 1.0, n)
        elif family == orc.GDN:
            a = rng.uniform(0.3, 1.0, n)
            b = rng.uniform(0.0, 1.0, n)
        else:
            a = rng.uniform(0.3, 1.0, (n, K))
            b = rng.uniform(0.0, 1.0, n)
        toks.append((k, v, a, b))
    return toks


def relerr(x, y):
    x, y = np.asarray(x, dtype=np.float64), np.asarray(y, dtype=np.float64)
    return np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300)


# ----------------------------------------------------------------------------
# 1. windowed form == step-by-step recurrence (paper §3.2: S_tau^T q = S0^T q~ + o_buf)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("family", FAMS)
@pytest.mark.parametrize("tau", [1, 2, 5, 16])
def test_window_read_equals_recurrence(family, tau):
    rng = np.random.default_rng(100 + 10 * family + tau)
    n, K, V = 6, 16, 12
    S0 = rng.standard_normal((n, K, V)) * 0.3
    toks = rand_tokens(rng, family, n, K, V, tau)
    q = rng.standard_normal((n, K))
    S, o_rec = orc.flush(family, S0, toks, q)
    o_win = orc.windowed_exact_output(family, S0, toks, q)
    assert relerr(o_win, o_rec) < 1e-12


# ----------------------------------------------------------------------------
# 2. brute force over exact rationals (dense explicit M_t)
# ----------------------------------------------------------------------------
def dyadic(rng, shape, lo=-8, hi=8, den=8):
    return rng.integers(lo, hi + 1, size=shape) / den


def frac(x):
    if np.ndim(x) == 0:
        return Fraction(float(x))
    return [frac(e) for e in x]


@pytest.mark.parametrize("family", FAMS)
@pytest.mark.parametrize("K,V,W", [(1, 1, 1), (2, 3, 2), (3, 2, 3), (4, 4, 4), (4, 1, 3)])
def test_bruteforce_exact_rationals(family, K, V, W):
    rng = np.random.default_rng(1000 + 100 * family + 10 * K + V + W)
    S0 = dyadic(rng, (K, V))
    toks, toks_f = [], []
    for _ in range(W):
        k = dyadic(rng, (K,), -4, 4, 4)
        v = dyadic(rng, (V,))
        b = rng.integers(0, 5) / 4.0
        a = (rng.integers(1, 9, size=K) / 8.0) if family == orc.KDA else rng.integers(1, 9) / 8.0
        toks.append((k[None], v[None], np.atleast_1d(a)[None] if family == orc.KDA else np.array([a]),
                     np.array([b])))
        toks_f.append((frac(k), frac(v), frac(a), Fraction(b)))
    qs = [dyadic(rng, (K,)) for _ in range(W)]
    states, outs = bf.recurrence(family, frac(S0), toks_f, [frac(q) for q in qs])
    # flush state and exact output after every prefix of the window
    for t in range(1, W + 1):
        S, o = orc.flush(family, S0[None], toks[:t], qs[t - 1][None])
        exact_S = np.array([[float(x) for x in r] for r in states[t - 1]])
        exact_o = np.array([float(x) for x in outs[t - 1]])
        assert np.allclose(S[0], exact_S, rtol=0, atol=1e-12 * max(1.0, np.abs(exact_S).max()))
        assert np.allclose(o[0], exact_o, rtol=0, atol=1e-12 * max(1.0, np.abs(exact_o).max()))
        # effective query and buffered term against the dense decomposition
        qt, ob = orc.effective_query(family, toks[:t], qs[t - 1][None])
        eq, eob = bf.window_decomposition(family, toks_f[:t], frac(qs[t - 1]))
        assert np.allclose(qt[0], [float(x) for x in eq], rtol=0, atol=1e-12)
        assert np.allclose(ob[0], [float(x) for x in eob], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# 3. Mamba-2 closed forms (paper §C.1: for Mamba-2, q~_t = d[t] ⊙ q_t)
# ----------------------------------------------------------------------------
def test_mamba2_effective_query_closed_form():
    rng = np.random.default_rng(7)
    n, K, V, tau = 5, 32, 8, 9
    toks = rand_tokens(rng, orc.MAMBA2, n, K, V, tau)
    q = rng.standard_normal((n, K))
    qt, ob = orc.effective_query(orc.MAMBA2, toks, q)
    d = np.prod(np.stack([t[2] for t in toks]), axis=0)        # product of every decay
    assert relerr(qt, d[:, None] * q) < 1e-14
    # buffered term: sum_j dt_j (prod_{i>j} a_i) (k_j . q) v_j
    ob_cf = np.zeros((n, V))
    for j, (k, v, a, b) in enumerate(toks):
        later = np.prod(np.stack([t[2] for t in toks[j + 1:]]), axis=0) if j + 1 < tau else np.ones(n)
        ob_cf += (b * later * np.sum(k * q, -1))[:, None] * v
    assert relerr(ob, ob_cf) < 1e-13


def test_mamba2_flush_closed_form():
    """Scalar decay: S_W = (prod a) S0 + sum_j (prod_{i>j} a_i) dt_j k_j v_j^T."""
    rng = np.random.default_rng(8)
    n, K, V, W = 4, 16, 8, 16
    S0 = rng.standard_normal((n, K, V))
    toks = rand_tokens(rng, orc.MAMBA2, n, K, V, W)
    S, _ = orc.flush(orc.MAMBA2, S0, toks)
    ref = np.prod(np.stack([t[2] for t in toks]), axis=0)[:, None, None] * S0
    for j, (k, v, a, b) in enumerate(toks):
        later = np.prod(np.stack([t[2] for t in toks[j + 1:]]), axis=0) if j + 1 < W else np.ones(n)
        ref += (b * later)[:, None, None] * np.einsum("nk,nv->nkv", k, v)
    assert relerr(S, ref) < 1e-13


def test_mamba2_transition_params():
    dt = np.array([0.0, 0.125, 1.5, 3.0])
    A = np.array([-0.5, -1.0, -2.0, -7.0])
    a, b = orc.transition_params(orc.MAMBA2, dt, None, A)
    import math
    assert np.all(b == dt)
    assert all(abs(a[i] - math.exp(dt[i] * A[i])) <= 4e-16 * math.exp(dt[i] * A[i]) for i in range(4))
    assert a[0] == 1.0            # zero decay rate -> identity transition


# ----------------------------------------------------------------------------
# 4. delta-rule write/read property
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("family", [orc.GDN, orc.KDA])
def test_delta_rule_overwrites_value_at_key(family):
    """With |k| = 1 the new state answers query k with the written value:
    GDN:  S_t^T k = (1-b) a S_{t-1}^T k + b v
    KDA:  S_t^T k = (1-b) (Diag(a) S_{t-1})^T k + b v
    and with a = 1, b = 1 the read returns v exactly (the delta rule replaces
    the value stored at key k)."""
    rng = np.random.default_rng(11)
    n, K, V = 7, 24, 10
    S = rng.standard_normal((n, K, V))
    (k, v, a, b), = rand_tokens(rng, family, n, K, V, 1)
    St = orc.update(family, S, k, v, a, b)
    got = orc.read(St, k)
    if family == orc.GDN:
        want = ((1 - b) * a)[:, None] * orc.read(S, k) + b[:, None] * v
    else:
        want = (1 - b)[:, None] * orc.read(a[:, :, None] * S, k) + b[:, None] * v
    assert relerr(got, want) < 1e-13
    ones = np.ones_like(a)
    St = orc.update(family, S, k, v, ones, np.ones(n))
    assert relerr(orc.read(St, k), v) < 1e-13


def test_kda_with_uniform_decay_is_gdn():
    rng = np.random.default_rng(12)
    n, K, V = 5, 16, 16
    S = rng.standard_normal((n, K, V))
    (k, v, a, b), = rand_tokens(rng, orc.GDN, n, K, V, 1)
    g = orc.update(orc.GDN, S, k, v, a, b)
    kd = orc.update(orc.KDA, S, k, v, np.repeat(a[:, None], K, 1), b)
    assert relerr(kd, g) < 1e-15


# ----------------------------------------------------------------------------
# 5. sketched read (project page, "Coefficient vector & readout")
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("family", FAMS)
def test_full_rank_identity_basis_reads_exactly(family):
    rng = np.random.default_rng(20 + family)
    n, K, V, tau = 4, 16, 8, 5
    S0 = rng.standard_normal((n, K, V))
    toks = rand_tokens(rng, family, n, K, V, tau)
    q = rng.standard_normal((n, K))
    qt, ob = orc.effective_query(family, toks, q)
    U = orc.sketch(S0, np.eye(K))
    o_hat = orc.sketched_output(U, np.eye(K), qt, ob)
    assert relerr(o_hat, orc.windowed_exact_output(family, S0, toks, q)) < 1e-13


def test_query_in_basis_span_reads_exactly():
    rng = np.random.default_rng(21)
    n, K, V, r = 3, 16, 8, 5
    Q, _ = np.linalg.qr(rng.standard_normal((K, K)))
    P = Q[:, :r]
    S0 = rng.standard_normal((n, K, V))
    qt = rng.standard_normal((n, r)) @ P.T
    ob = rng.standard_normal((n, V))
    o_hat = orc.sketched_output(orc.sketch(S0, P), P.T, qt, ob)
    assert relerr(o_hat, orc.read(S0, qt) + ob) < 1e-13


def test_sketch_error_is_projection_residual():
    """With C = P^T (orthonormal P): o - o^ = S0^T (I - P P^T) q~."""
    rng = np.random.default_rng(22)
    n, K, V, r = 4, 16, 8, 6
    Q, _ = np.linalg.qr(rng.standard_normal((K, K)))
    P = Q[:, :r]
    S0 = rng.standard_normal((n, K, V))
    qt = rng.standard_normal((n, K))
    ob = np.zeros((n, V))
    err = orc.read(S0, qt) - orc.sketched_output(orc.sketch(S0, P), P.T, qt, ob)
    resid = qt - (qt @ P) @ P.T
    assert relerr(err, orc.read(S0, resid)) < 1e-12
    # the columns of the sketch are the state's answers to the basis vectors
    U = orc.sketch(S0, P)
    for i in range(r):
        assert relerr(U[..., i], orc.read(S0, np.broadcast_to(P[:, i], (n, K)))) < 1e-14


# ----------------------------------------------------------------------------
# 6. flush identities (zero buffer / zero decay give the identity)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("family", FAMS)
def test_flush_identity_bit_exact(family):
    rng = np.random.default_rng(30 + family)
    n, K, V, W = 3, 16, 8, 6
    S0 = rng.standard_normal((n, K, V))
    toks = rand_tokens(rng, family, n, K, V, W)
    ident = [(k, v, np.ones_like(a), np.zeros_like(b)) for (k, v, a, b) in toks]
    S, _ = orc.flush(family, S0, ident)
    assert np.array_equal(S, S0)
    S, _ = orc.flush(family, S0, [])
    assert np.array_equal(S, S0)


# ----------------------------------------------------------------------------
# 7. schedule: W-1 non-flush steps then a flush (paper App. B)
# ----------------------------------------------------------------------------
def session_inputs(rng, family, B, H, K, V):
    def bits(x):
        import torch
        return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    k = rng.standard_normal((B, H, K)) / np.sqrt(K)
    q = rng.standard_normal((B, H, K)) / np.sqrt(K)
    if family != orc.MAMBA2:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    gate = (rng.uniform(0.05, 1.0, (B, H)) if family != orc.KDA else rng.uniform(0.3, 1.0, (B, H, K)))
    return {"q": bits(q), "k": bits(k), "v": bits(rng.standard_normal((B, H, V))),
            "gate": gate.astype(np.float32), "beta": rng.uniform(0, 1, (B, H)).astype(np.float32)}


@pytest.mark.parametrize("family", FAMS)
def test_session_modes_agree_at_window_boundaries(family):
    rng = np.random.default_rng(40 + family)
    B, H, K, V, W, T = 2, 3, 8, 6, 4, 12
    S0 = rng.standard_normal((B, H, K, V))
    A = -np.exp(rng.uniform(0, 2, H))
    offs = np.array([0, 2, 3, 6])
    basis = rng.standard_normal((6, K))
    sk = orc.Session(family, S0, W, A, basis, basis, offs)
    rp = orc.Session(family, S0, W, A)
    st = orc.Session(family, S0, W, A)
    sk.prime()
    for t in range(1, T + 1):
        inp = session_inputs(rng, family, B, H, K, V)
        o_std = st.exact_step(inp)
        if t % W == 0:
            assert sk.phase == W - 1 and rp.phase == W - 1
            o_sk = sk.flush(inp)
            o_rp = rp.flush(inp, with_sketch=False)
            assert relerr(o_sk, o_std) < 1e-12 and relerr(o_rp, o_std) < 1e-12
            assert relerr(sk.S, st.S) < 1e-12 and relerr(rp.S, st.S) < 1e-12
            assert sk.phase == 0
        else:
            assert sk.phase == (t - 1) % W
            _, o_exact = sk.decode(inp)
            o_rp = rp.replay_step(inp)
            assert relerr(o_exact, o_std) < 1e-12 and relerr(o_rp, o_std) < 1e-12


# ----------------------------------------------------------------------------
# 8. number formats against torch's own conversions
# ----------------------------------------------------------------------------
def test_bf16_widen_and_round_match_torch():
    import torch
    rng = np.random.default_rng(50)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 - 2.0 ** -9,
                         2.0 ** -130, 3.0 * 2.0 ** -134, 3.3e38, -3.4e38]]).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.widen_bf16(bits), t.to(torch.float64).numpy())
    got = orc.round_bf16(x.astype(np.float64))
    want = t.to(torch.float64).numpy()
    assert np.array_equal(got, want)
    # ties go to even: 1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    assert orc.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert orc.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6


# ----------------------------------------------------------------------------
# 9. the synthetic generator's distributions (not the method: a sanity pin)
# ----------------------------------------------------------------------------
def test_synth_ranks_and_basis():
    from ssm_decode_b200 import synth
    wl = synth.WORKLOADS["mamba2_b320"]
    st = synth.static_inputs(synth.shrink(wl, batch=1), with_state=False)
    assert st.ranks.sum() == 8 * wl.heads and st.ranks.min() >= 2 and st.ranks.max() <= 16
    h = 3
    P = st.basis[st.offsets[h]:st.offsets[h + 1]].astype(np.float64)
    assert np.allclose(P @ P.T, np.eye(len(P)), atol=1e-6)
    # the basis is the top eigenvectors of the query covariance G G^T + 0.01 I
    G = st.qmix[h].astype(np.float64)
    w, vec = np.linalg.eigh(G @ G.T + 0.01 * np.eye(wl.dk))
    top = vec[:, ::-1][:, :len(P)]
    assert np.allclose(np.abs(top.T @ P.T), np.eye(len(P)), atol=1e-4)


# ----------------------------------------------------------------------------
# 9b. state-dependent coefficient map (project page, "Per window · Flush:
#     Sketch & coefficient map", C = (U^T U)^+ U^T S0^T; paper §A.2.1: the
#     coefficients minimise ||S0^T q~ - U c||_2)
# ----------------------------------------------------------------------------
def _map_case(seed, n=4, K=12, V=20, r=5):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((n, K, V))
    P = np.linalg.qr(rng.standard_normal((K, K)))[0][:, :r]
    q = rng.standard_normal((n, K))
    return S, P, orc.sketch(S, P), q


def test_coefficient_map_is_least_squares():
    """c = C q~ is numpy's least-squares solution of min_c ||S^T q~ - U c||."""
    S, P, U, q = _map_case(1)
    C = orc.coefficient_map(U, S)
    for i in range(len(S)):
        c_ls = np.linalg.lstsq(U[i], S[i].T @ q[i], rcond=None)[0]
        assert relerr(C[i] @ q[i], c_ls) < 1e-10


def test_coefficient_map_residual_is_orthogonal_to_sketch():
    """Normal equations: the readout error S^T q~ - U C q~ is orthogonal to every u_i."""
    S, P, U, q = _map_case(2, K=16, V=9, r=6)
    C = orc.coefficient_map(U, S)
    res = np.einsum("nkv,nk->nv", S, q) - np.einsum("nvr,nrk,nk->nv", U, C, q)
    assert np.abs(np.einsum("nvr,nv->nr", U, res)).max() < 1e-10 * np.abs(res).max()


def test_coefficient_map_full_rank_is_identity():
    """r = K <= V with a square orthogonal basis P: U = S^T P has full column
    rank, so C = (P^T S S^T P)^{-1} P^T S S^T = P^T and every read is exact."""
    S, P, U, q = _map_case(3, K=8, V=20, r=8)
    C = orc.coefficient_map(U, S)
    assert relerr(C, np.broadcast_to(P.T, C.shape)) < 1e-10
    o = np.einsum("nkv,nk->nv", S, q)
    assert relerr(orc.sketched_output(U, C, q, 0.0), o) < 1e-10


def test_coefficient_map_ridge_is_augmented_least_squares():
    """With the ridge, c = C q~ solves min ||S^T q~ - U c||^2 + lambda ||c||^2,
    lambda = rho tr(U^T U) / r: the stacked system [U; sqrt(lambda) I] c ~ [S^T q~; 0]."""
    S, P, U, q = _map_case(4)
    rho = 0.3
    C = orc.coefficient_map(U, S, rho)
    r = U.shape[-1]
    for i in range(len(S)):
        lam = rho * np.sum(U[i] * U[i]) / r
        A = np.vstack([U[i], np.sqrt(lam) * np.eye(r)])
        y = np.concatenate([S[i].T @ q[i], np.zeros(r)])
        assert relerr(C[i] @ q[i], np.linalg.lstsq(A, y, rcond=None)[0]) < 1e-10


def test_state_map_never_worse_than_fixed_map():
    """The least-squares map reads at least as well as the fixed C = P^T."""
    S, P, U, q = _map_case(5, K=32, V=16, r=6)
    o = np.einsum("nkv,nk->nv", S, q)
    e_state = np.linalg.norm(o - orc.sketched_output(U, orc.coefficient_map(U, S), q, 0.0), axis=-1)
    e_fixed = np.linalg.norm(o - orc.sketched_output(U, P.T, q, 0.0), axis=-1)
    assert (e_state <= e_fixed * (1 + 1e-12)).all() and (e_state < e_fixed).any()


def test_coefficient_map_of_zero_state_is_zero():
    """No positive-definite Gram matrix (U = 0): the map is zero, so the
    sketched read returns only the exact buffered term."""
    S = np.zeros((2, 8, 6))
    P = np.eye(8)[:, :3]
    assert not orc.coefficient_map(orc.sketch(S, P), S, 0.5).any()


def test_lrd_map_with_every_column_kept_is_the_exact_map():
    """n_piv = V keeps every output column: H^ = H and the map is the exact one."""
    S, P, U, q = _map_case(7, K=10, V=6, r=4)
    for rho in (0.0, 0.2):
        assert relerr(orc.coefficient_map_lrd(S, P, n_piv=6, rho=rho), orc.coefficient_map(U, S, rho)) < 1e-10


def test_lrd_map_of_isotropic_energy_is_the_fixed_map():
    """No pivots and equal coordinate-wise energy (H^ = cI): with an orthonormal
    basis the map is P^T, the fixed map."""
    K, V, r = 8, 16, 3
    rng = np.random.default_rng(8)
    Q = np.linalg.qr(rng.standard_normal((V, V)))[0][:K]        # orthonormal rows: S S^T = I
    S = np.stack([2.0 * Q, 0.5 * Q])
    P = np.linalg.qr(rng.standard_normal((K, K)))[0][:, :r]
    C = orc.coefficient_map_lrd(S, P, n_piv=0)
    assert relerr(C, np.broadcast_to(P.T, C.shape)) < 1e-10


def test_lrd_map_matches_a_direct_construction():
    """Against H^ built column by column from its definition (pivots by energy,
    diagonal of the rest) and a least-squares solve in the H^ metric."""
    S, P, U, q = _map_case(9, n=2, K=7, V=9, r=3)
    C = orc.coefficient_map_lrd(S, P, n_piv=2)
    for i in range(len(S)):
        e = [float(S[i][:, v] @ S[i][:, v]) for v in range(S.shape[2])]
        piv = sorted(range(len(e)), key=lambda v: -e[v])[:2]
        H = sum(np.outer(S[i][:, v], S[i][:, v]) for v in piv)
        H = H + np.diag(sum(S[i][:, v] ** 2 for v in range(len(e)) if v not in piv))
        # c minimises (q - P c)^T H (q - P c): weighted least squares via a square root of H
        w, Qh = np.linalg.eigh(H)
        Hh = Qh @ np.diag(np.sqrt(np.maximum(w, 0))) @ Qh.T
        c_ls = np.linalg.lstsq(Hh @ P, Hh @ q[i], rcond=None)[0]
        assert relerr(C[i] @ q[i], c_ls) < 1e-8


def test_lrd_map_of_a_state_on_few_columns_is_the_exact_map():
    """A state whose energy sits in at most n_piv output columns: those columns
    are the pivots, the rest is zero (D = 0), so H^ = H and the map is exact."""
    S, P, U, q = _map_case(10, n=3, K=9, V=12, r=3)
    S = S.copy()
    S[0][:, [0, 1, 2, 4, 6, 7, 8, 9, 11]] = 0.0          # columns 3, 5, 10 remain
    S[1][:, :-4] = 0.0                                     # the last four remain
    S[2][:, 4:] = 0.0                                      # the first four remain,
    S[2][:, 0] *= 50.0                                     # one of them dominant
    U = orc.sketch(S, P)
    for rho in (0.0, 0.1):
        C = orc.coefficient_map_lrd(S, P, n_piv=4, rho=rho)
        assert relerr(C, orc.coefficient_map(U, S, rho)) < 1e-10


def test_lrd_map_ties_keep_the_lower_column():
    """Equal energies rank the lower column first (the pages leave ties open;
    this is the stable ranking the kernel shares): with one pivot and columns 1
    and 3 tied for the largest energy, H^ = s1 s1^T + diag(s3^2 + rest)."""
    rng = np.random.default_rng(11)
    K, r = 6, 2
    S = np.zeros((K, 5))
    S[:, 1] = rng.standard_normal(K)
    S[:, 3] = S[:, 1] * np.array([1, -1, 1, 1, -1, 1])    # same squares: an exact tie
    S[:, 0] = 0.1 * rng.standard_normal(K)
    P = np.linalg.qr(rng.standard_normal((K, K)))[0][:, :r]
    H = np.outer(S[:, 1], S[:, 1]) + np.diag(S[:, 0] ** 2 + S[:, 3] ** 2)
    want = np.linalg.solve(P.T @ H @ P, P.T @ H)
    assert relerr(orc.coefficient_map_lrd(S, P, n_piv=1), want) < 1e-10
    # the other choice is a different map: the pin can tell them apart
    H3 = np.outer(S[:, 3], S[:, 3]) + np.diag(S[:, 0] ** 2 + S[:, 1] ** 2)
    assert relerr(np.linalg.solve(P.T @ H3 @ P, P.T @ H3), want) > 1e-3


@pytest.mark.parametrize("family", FAMS)
def test_session_state_map_identity_basis_reads_exactly(family):
    """Session with the state map and P = I (r = K <= V): every sketched read
    equals the exact windowed read (C = I)."""
    from ssm_decode_b200 import synth
    rng = np.random.default_rng(6)
    B, H, K, V, W = 2, 2, 4, 6, 4
    S0 = rng.standard_normal((B, H, K, V))
    offsets = np.arange(H + 1) * K
    basis = np.tile(np.eye(K), (H, 1))
    A = -np.exp(rng.uniform(0, 1, H))
    sess = orc.Session(family, S0, W, A, basis, basis, offsets, state_map=True)
    sess.prime()
    for _ in range(W - 1):
        inp = {"q": synth.f32_to_bf16_bits(rng.standard_normal((B, H, K))),
               "k": synth.f32_to_bf16_bits(rng.standard_normal((B, H, K)) / 2),
               "v": synth.f32_to_bf16_bits(rng.standard_normal((B, H, V))),
               "gate": (rng.uniform(0.2, 0.9, (B, H, K)) if family == orc.KDA
                        else rng.uniform(0.2, 0.9, (B, H))),
               "beta": rng.uniform(0.1, 0.9, (B, H))}
        o_hat, o = sess.decode(inp)
        assert relerr(o_hat, o) < 1e-9


# ----------------------------------------------------------------------------
# 10. planted mistakes must fail a pin
# ----------------------------------------------------------------------------
def _run_pins():
    """Run the pins that exercise the recurrence; return True if all pass."""
    try:
        for fam in FAMS:
            for tau in (1, 5):
                test_window_read_equals_recurrence(fam, tau)
            test_bruteforce_exact_rationals(fam, 3, 2, 3)
            test_full_rank_identity_basis_reads_exactly(fam)
        test_mamba2_effective_query_closed_form()
        test_mamba2_flush_closed_form()
        for fam in (orc.GDN, orc.KDA):
            test_delta_rule_overwrites_value_at_key(fam)
        test_kda_with_uniform_decay_is_gdn()
        test_sketch_error_is_projection_residual()
    except AssertionError:
        return False
    return True


def _run_map_pins():
    try:
        test_coefficient_map_is_least_squares()
        test_coefficient_map_residual_is_orthogonal_to_sketch()
        test_coefficient_map_full_rank_is_identity()
        test_coefficient_map_ridge_is_augmented_least_squares()
        test_state_map_never_worse_than_fixed_map()
    except AssertionError:
        return False
    return True


ORIG_MAP = orc.coefficient_map
ORIG_LRD = orc.coefficient_map_lrd


def _mut_lrd_no_diagonal(S, P, n_piv=4, rho=0.0):
    # keeps only the pivot columns: the remaining coordinate-wise energy is dropped
    e = np.einsum("...kv,...kv->...v", S, S)
    keep = np.argsort(-e, axis=-1, kind="stable")[..., :n_piv]
    mask = np.zeros(e.shape, bool)
    np.put_along_axis(mask, keep, True, axis=-1)
    return ORIG_LRD(S * mask[..., None, :], P, n_piv, rho)


def _lrd_variant(S, P, n_piv, rho, smallest=False, diag_all=False, ridge_of_h=False,
                 ties_high=False):
    """The low-rank-plus-diagonal map with one plausible mistake switched on."""
    S = np.asarray(S, np.float64)
    K, r = S.shape[-2], P.shape[-1]
    e = np.einsum("...kv,...kv->...v", S, S)
    key = e if smallest else -e
    if ties_high:
        order = S.shape[-1] - 1 - np.argsort(key[..., ::-1], axis=-1, kind="stable")
    else:
        order = np.argsort(key, axis=-1, kind="stable")
    piv = order[..., :n_piv]
    mask = np.zeros(e.shape, bool)
    np.put_along_axis(mask, piv, True, axis=-1)
    L = S * mask[..., None, :]
    d = np.einsum("...kv,...kv->...k", S if diag_all else S * ~mask[..., None, :], S)
    H = np.einsum("...kp,...jp->...kj", L, L) + d[..., :, None] * np.eye(K)
    G = np.einsum("kr,...kj,js->...rs", P, H, P)
    tr = np.trace(H if ridge_of_h else G, axis1=-2, axis2=-1)
    A = G + (rho * tr / r)[..., None, None] * np.eye(r)
    return np.linalg.solve(A, np.einsum("kr,...kj->...rj", P, H))


def _run_lrd_pins():
    try:
        test_lrd_map_with_every_column_kept_is_the_exact_map()
        test_lrd_map_of_isotropic_energy_is_the_fixed_map()
        test_lrd_map_matches_a_direct_construction()
        test_lrd_map_of_a_state_on_few_columns_is_the_exact_map()
        test_lrd_map_ties_keep_the_lower_column()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("mutant", [
    _mut_lrd_no_diagonal,
    lambda S, P, n_piv=4, rho=0.0: _lrd_variant(S, P, n_piv, rho, smallest=True),
    lambda S, P, n_piv=4, rho=0.0: _lrd_variant(S, P, n_piv, rho, diag_all=True),
    lambda S, P, n_piv=4, rho=0.0: _lrd_variant(S, P, n_piv, rho, ridge_of_h=True),
    lambda S, P, n_piv=4, rho=0.0: _lrd_variant(S, P, n_piv, rho, ties_high=True),
], ids=["no_diagonal", "smallest_pivots", "diagonal_of_all", "ridge_of_H", "ties_high"])
def test_planted_lrd_mistakes_are_caught(monkeypatch, mutant):
    assert _run_lrd_pins()
    monkeypatch.setattr(orc, "coefficient_map_lrd", lambda S, P, n_piv=4, rho=0.0: _lrd_variant(S, P, n_piv, rho))
    assert _run_lrd_pins(), "the mutant harness itself must pass unmutated"
    monkeypatch.setattr(orc, "coefficient_map_lrd", mutant)
    assert not _run_lrd_pins(), "a mistake planted in coefficient_map_lrd went unnoticed"


def _mut_map_no_ridge(U, S, rho=0.0):
    return ORIG_MAP(U, S, 0.0)


def _mut_map_sign(U, S, rho=0.0):
    return -ORIG_MAP(U, S, rho)


def _mut_map_gram_only(U, S, rho=0.0):
    # skips the Gram solve: C = U^T S^T
    return np.einsum("...vr,...kv->...rk", U, S)


@pytest.mark.parametrize("mutant", [_mut_map_no_ridge, _mut_map_sign, _mut_map_gram_only])
def test_planted_map_mistakes_are_caught(monkeypatch, mutant):
    assert _run_map_pins()
    monkeypatch.setattr(orc, "coefficient_map", mutant)
    assert not _run_map_pins(), "a mistake planted in coefficient_map went unnoticed"


def _mut_erase_sign(family, x, k, a, b):
    if family == orc.MAMBA2:
        return a[..., None] * x
    kx = np.einsum("...k,...k->...", k, x)
    erased = x + (b * kx)[..., None] * k
    return a[..., None] * erased if family == orc.GDN else a * erased


def _mut_kda_order(family, S, k, a, b):
    if family != orc.KDA:
        return ORIG_APPLY(family, S, k, a, b)
    ktS = np.einsum("...k,...kv->...v", k, S)
    return a[..., :, None] * (S - b[..., None, None] * k[..., :, None] * ktS[..., None, :])


def _mut_drop_buffer_term(family, tokens, q):
    qt, ob = ORIG_EQ(family, tokens, q)
    return qt, ob - ob   # dropped exact buffered term


def _mut_sketch_transposed(S, P):
    return np.einsum("...kv,kr->...vr", S, P[::-1])


def _mut_decay_twice(family, x, k, a, b):
    y = ORIG_APPLY_T(family, x, k, a, b)
    return a[..., None] * y if family == orc.MAMBA2 else y


ORIG_APPLY = orc.apply_transition
ORIG_APPLY_T = orc.apply_transition_T
ORIG_EQ = orc.effective_query


@pytest.mark.parametrize("target,mutant", [
    ("apply_transition_T", _mut_erase_sign),
    ("apply_transition", _mut_kda_order),
    ("effective_query", _mut_drop_buffer_term),
    ("sketch", _mut_sketch_transposed),
    ("apply_transition_T", _mut_decay_twice),
])
def test_planted_mistakes_are_caught(monkeypatch, target, mutant):
    assert _run_pins()
    monkeypatch.setattr(orc, target, mutant)
    assert not _run_pins(), f"a mistake planted in {target} went unnoticed"


# ----------------------------------------------------------------------------
# 11. the pages' printed traffic figures (golden fixture)
# ----------------------------------------------------------------------------
def test_golden_traffic_fixture_is_well_formed():
    with open(os.path.join(GOLDEN, "traffic_reduction.json")) as f:
        g = json.load(f)
    assert {c["name"] for c in g["cases"]} >= {"mamba2_r8", "mamba2_r4", "gdn_r8", "gdn_r4", "replay"}
    for c in g["cases"]:
        assert c["citation"]
