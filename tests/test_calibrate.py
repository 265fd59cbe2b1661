"""Offline calibration (ssm_decode_b200/calibrate.py) against closed forms,
brute force and the synthetic generator's own basis.  CPU only.

Basis (project page, "Offline · Fixed: Sketching matrix"; paper §A.1):
Omega* = E0^{-1/2} P_G minimises L_G(Omega) = E min_c ||E0^{1/2}(q~ - Omega c)||^2.
Ranks (paper §4.2, App. E): knapsack over per-head options by a bisected
traffic price, then slack filling.
"""
import itertools

import numpy as np
import pytest

from ssm_decode_b200 import calibrate as cal
from ssm_decode_b200 import synth


def _samples(seed, N=40, M=400, K=8, V=12):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((K, K)) * np.linspace(1.5, 0.3, K)      # anisotropic states
    S = np.einsum("kj,njv->nkv", A, rng.standard_normal((N, K, V)))
    B = rng.standard_normal((K, K)) * np.linspace(2.0, 0.1, K)
    q = rng.standard_normal((M, K)) @ B.T
    return S, q


def _loss(Omega, E0, q):
    """L(Omega) with the optimal c for each q (weighted least squares)."""
    if Omega.shape[1] == 0:
        return float(np.mean(np.einsum("mk,kj,mj->m", q, E0, q)))
    M = Omega.T @ E0 @ Omega
    c = np.linalg.solve(M, Omega.T @ E0 @ q.T).T
    d = q - c @ Omega.T
    return float(np.mean(np.einsum("mk,kj,mj->m", d, E0, d)))


def test_basis_loss_is_the_energy_tail():
    """Eckart-Young in the E0 metric: the loss of the rank-r basis is the sum of
    the trailing eigenvalues of E[z z^T], and the fixed map C* attains it."""
    S, q = _samples(1)
    hb = cal.fit_head_basis(S, q)
    tails = cal.loss_curve(hb, range(9))
    for r in range(9):
        assert abs(_loss(hb.omega[:, :r], hb.E0, q) - tails[r]) <= 1e-9 * max(tails[0], 1)
        assert abs(cal.reconstruction_error(hb, S, q, r) - tails[r]) <= 1e-9 * max(tails[0], 1)
    assert tails[-1] == 0 and np.all(np.diff(tails) <= 1e-12)


def test_basis_beats_random_bases():
    S, q = _samples(2)
    hb = cal.fit_head_basis(S, q)
    rng = np.random.default_rng(3)
    for r in (1, 3, 5):
        best = _loss(hb.omega[:, :r], hb.E0, q)
        for _ in range(200):
            assert _loss(rng.standard_normal((8, r)), hb.E0, q) >= best * (1 - 1e-9)


def test_fixed_map_is_the_optimal_coefficients():
    """c = C* q~ equals the weighted least-squares coefficients of Omega*."""
    S, q = _samples(4)
    hb = cal.fit_head_basis(S, q)
    r = 4
    Om = hb.omega[:, :r]
    c_opt = np.linalg.solve(Om.T @ hb.E0 @ Om, Om.T @ hb.E0 @ q.T).T
    assert np.allclose(q @ hb.coef[:r].T, c_opt, atol=1e-9 * np.abs(c_opt).max())
    assert np.allclose(Om.T @ hb.E0 @ Om, np.eye(r), atol=1e-9)


def test_isotropic_states_recover_the_generators_basis():
    """With the generator's states (iid, E0 ~ 0.1 dv I) and its structured
    queries q = G z + 0.1 n, the calibrated subspace is the generator's own
    basis P_h = Q_h[:, :r_h] (top eigenvectors of G G^T + 0.01 I)."""
    wl = synth.Workload("cal", synth.GDN, 64, 2, 64, 64, 16, 0, 6, 9, ragged=False, structured_q=True)
    st = synth.static_inputs(wl)
    h = 1
    q = np.concatenate([synth.bf16_bits_to_f32(synth.step_inputs(wl, st, t)["q"][:, h]) for t in range(60)])
    hb = cal.fit_head_basis(st.state[:, h], q)
    r = int(st.ranks[h])
    P = st.basis[st.offsets[h]:st.offsets[h + 1]].T.astype(np.float64)        # [K, r], orthonormal
    Om = np.linalg.qr(hb.omega[:, :r])[0]
    # principal angles: the smallest singular value of P^T Om near 1
    assert np.linalg.svd(P.T @ Om, compute_uv=False).min() > 0.97


def _brute(scores, costs, budget):
    best = (np.inf, None)
    for ch in itertools.product(*[range(scores.shape[1])] * len(scores)):
        ch = np.array(ch)
        t = costs[np.arange(len(ch)), ch].sum()
        s = scores[np.arange(len(ch)), ch].sum()
        if t <= budget and s < best[0]:
            best = (s, ch)
    return best


def test_allocation_matches_brute_force_on_convex_heads():
    """Convex decreasing errors, equal-cost rank steps: price + slack is optimal."""
    rng = np.random.default_rng(5)
    for _ in range(30):
        H, R = 4, 5
        decay = rng.uniform(0.3, 0.9, (H, 1))
        scores = rng.uniform(0.5, 3.0, (H, 1)) * decay ** np.arange(1, R + 1)
        costs = np.broadcast_to(np.arange(1, R + 1, dtype=float), (H, R)).copy()
        budget = float(rng.integers(H, H * R + 1))
        ch = cal.allocate(scores, costs, budget)
        assert costs[np.arange(H), ch].sum() <= budget
        assert scores[np.arange(H), ch].sum() <= _brute(scores, costs, budget)[0] * (1 + 1e-9)


def test_allocation_with_dense_option_is_feasible_and_beats_uniform():
    rng = np.random.default_rng(6)
    K, V, W = 128, 64, 16
    for _ in range(20):
        H = 6
        err = np.sort(rng.uniform(0, 1, (H, 17)), axis=1)[:, ::-1] * rng.uniform(0.1, 10, (H, 1))
        sens = rng.uniform(0.5, 2.0, H)
        a = cal.allocate_ranks(err, sens, K, V, W, mean_rank=8)
        budget = H * cal.traffic_per_step(8, K, V, W)
        assert a.traffic <= budget * (1 + 1e-12)
        uniform = float((sens * err[:, 8]).sum())
        assert a.score <= uniform * (1 + 1e-12)
        # small instance: brute force over ranks 1..4 and dense
        e4 = err[:3, :5]
        b = cal.allocate_ranks(e4, sens[:3], K, V, W, mean_rank=3, max_rank=4)
        scores = np.concatenate([sens[:3, None] * e4[:, 1:5], np.zeros((3, 1))], axis=1)
        costs = np.array([[cal.traffic_per_step(r, K, V, W) for r in range(1, 5)]
                          + [cal.traffic_per_step(0, K, V, W, dense=True)]] * 3)
        opt = _brute(scores, costs, 3 * cal.traffic_per_step(3, K, V, W))[0]
        assert b.score <= opt * 1.10 + 1e-12            # price + slack: within 10 % of optimal here
        assert b.traffic <= 3 * cal.traffic_per_step(3, K, V, W) * (1 + 1e-12)


def test_allocation_favours_sensitive_high_error_heads():
    """Heads with larger sensitivity x error get larger ranks (App. E)."""
    H = 8
    base = 0.8 ** np.arange(17)
    err = np.outer(np.linspace(0.2, 3.0, H), base)
    a = cal.allocate_ranks(err, np.ones(H), 128, 128, 16, mean_rank=8, dense=False)
    assert np.all(np.diff(a.ranks) >= 0) and a.ranks[-1] > a.ranks[0]


def test_budget_below_cheapest_is_refused():
    with pytest.raises(ValueError):
        cal.allocate(np.ones((2, 2)), np.ones((2, 2)), 1.0)


def test_calibration_feeds_the_library():
    """Bases and ranks calibrated on a synthetic model are valid library input:
    the plan accepts the ranks and dense flags, its buffers hold the packed
    basis and map rows, and the oracle's sketched read with the calibrated
    basis and map has the error the calibration predicted."""
    from oracle import sketchssm_oracle as orc
    from ssm_decode_b200 import binding as B
    from ssm_decode_b200 import build
    build.build()
    wl = synth.Workload("calpipe", synth.GDN, 24, 6, 64, 64, 16, 0, 8, 11)
    st = synth.static_inputs(wl)
    q = np.stack([synth.bf16_bits_to_f32(synth.step_inputs(wl, st, t)["q"]) for t in range(20)])   # [T, B, H, K]
    bases, errors = [], []
    for h in range(wl.heads):
        hb = cal.fit_head_basis(st.state[:, h], q[:, :, h].reshape(-1, wl.dk))
        bases.append(hb)
        errors.append([cal.reconstruction_error(hb, st.state[:, h], q[:, :, h].reshape(-1, wl.dk), r)
                       for r in range(17)])
    sens = np.random.default_rng(12).uniform(0.5, 2.0, wl.heads)
    alloc = cal.allocate_ranks(np.array(errors), sens, wl.dk, wl.dv, wl.window, mean_rank=8)
    dense = alloc.ranks == cal.DENSE
    ranks = np.where(dense, wl.dk, alloc.ranks).astype(np.int32)
    basis = np.concatenate([np.eye(wl.dk) if dense[h] else bases[h].omega[:, :ranks[h]].T
                            for h in range(wl.heads)]).astype(np.float32)
    coef = np.concatenate([np.eye(wl.dk) if dense[h] else bases[h].coef[:ranks[h]]
                           for h in range(wl.heads)]).astype(np.float32)
    plan = B.Plan(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, wl.window, ranks, B.SS_BF16,
                  dense_heads=dense.astype(np.uint8))
    sizes = B.ss_buffer_sizes(plan)
    assert sizes["total_rank"] == ranks.sum() == len(basis) == len(coef)
    assert sizes["basis"] == basis.nbytes and sizes["coef"] == coef.nbytes
    # the oracle reads with the calibrated basis and map: error as predicted
    offs = np.concatenate([[0], np.cumsum(ranks)])
    sess = orc.Session(wl.family, st.state, wl.window, None, basis, coef, offs, dense=dense)
    sess.prime()
    qt = q[0]                                           # no buffered updates: q~ = q
    for h in range(wl.heads):
        if dense[h]:
            continue
        o = np.einsum("bkv,bk->bv", st.state[:, h], qt[:, h])
        o_hat = orc.sketched_output(sess.U[h], sess.C[h], qt[:, h], 0.0)
        got = np.mean(np.sum((o - o_hat) ** 2, axis=-1))
        hb = bases[h]
        # the same error from the calibration side, on these states and queries
        proj = hb.omega[:, :ranks[h]] @ hb.coef[:ranks[h]]
        d = qt[:, h] - qt[:, h] @ proj.T
        want = np.mean(np.einsum("bk,bkv,bjv,bj->b", d, st.state[:, h], st.state[:, h], d))
        assert abs(got - want) <= 1e-6 * max(want, 1e-12) + 1e-9
