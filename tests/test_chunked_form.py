"""The chunked (WY) form of the delta-rule flush, and its TF32 precision plan,
against the oracle's step-by-step recurrence.  CPU only.

A flush applies W delta-rule updates to the state (project page, "Full state";
paper §4.1 and App. B).  Written without rescaling, with the running decay
products g_t = a_1 .. a_t (per channel, G_t, for KDA):

  GDN  S_W = g_W S_0 + sum_t (g_W / g_t) k_t w_t^T,
       w_t = b_t (v_t - g_t S_0^T k_t - sum_{j<t} (g_t / g_j)(k_t . k_j) w_j)
  KDA  S_W = Diag(G_W) S_0 + sum_t (k_t . G_W / G_t) w_t^T,
       w_t = b_t (v_t - S_0^T (G_t . k_t) - sum_{j<t} [sum_c k_t[c] k_j[c] G_t[c] / G_j[c]] w_j)

so the flush is three contractions per head (Y = S_0^T K, the rank-W update,
the read-out S_W^T [Omega | q]) around a W-step recursion on V-vectors.  Every
decay factor is a ratio <= 1.  These tests pin the identity in fp64 and the
split-operand scheme that keeps it at fp32 accuracy with TF32 products
(x = hi + lo, hi = x with its 13 low mantissa bits cleared): the scheme must
meet the 1e-4 parity bar with a wide margin, and dropping the third product
of the read-out must not.
"""
import numpy as np
import pytest

from oracle import sketchssm_oracle as orc


def _ratio(a, t, j):
    """prod_{i=j+1..t} a_i (scalar or per channel), 1 for t == j."""
    r = np.ones_like(a[0], dtype=np.float64)
    for i in range(j + 1, t + 1):
        r = r * a[i]
    return r


def chunked_flush(fam, S0, ks, vs, a, b, mm=None, split_b_read=True):
    """The chunked form.  mm(A, B, exact_b) computes A @ B; the default is fp64."""
    if mm is None:
        def mm(A, B, exact_a=False, exact_b=False, third=True):
            return A @ B
    W, K = ks.shape
    gdn = fam == orc.GDN
    gam = [_ratio(a, t, -1) for t in range(W)]                       # g_t (or G_t), 0-based t
    kread = ks if gdn else np.stack([gam[t] * ks[t] for t in range(W)])
    Y = mm(S0.T, kread.T, exact_b=gdn)                               # [V, W]
    w = np.zeros((W, S0.shape[1]))
    for t in range(W):
        acc = vs[t] - (gam[t] if gdn else 1.0) * Y[:, t]
        for j in range(t):
            pair = _ratio(a, t, j) * (ks[t] @ ks[j]) if gdn else np.sum(ks[t] * ks[j] * _ratio(a, t, j))
            acc = acc - pair * w[j]
        w[t] = b[t] * acc
    if gdn:
        wt = np.stack([_ratio(a, W - 1, t) * w[t] for t in range(W)])
        D = mm(ks.T, wt, exact_a=True)
        SW = gam[-1] * S0 + D
    else:
        kw = np.stack([ks[t] * _ratio(a, W - 1, t) for t in range(W)])
        D = mm(kw.T, w)
        SW = gam[-1][:, None] * S0 + D
    return SW


def _case(fam, seed, W=16, K=64, V=48, lo=0.85):
    rng = np.random.default_rng(seed)
    ks = rng.standard_normal((W, K))
    ks /= np.linalg.norm(ks, axis=1, keepdims=True)
    vs = rng.standard_normal((W, V))
    a = rng.uniform(lo, 1.0, W) if fam == orc.GDN else np.exp(rng.uniform(np.log(lo), 0.0, (W, K)))
    b = rng.uniform(0.1, 1.0, W)
    S0 = rng.standard_normal((K, V)) * np.sqrt(0.1)
    return S0, ks, vs, a, b


@pytest.mark.parametrize("fam", [orc.GDN, orc.KDA])
@pytest.mark.parametrize("lo", [0.85, 1e-3])
def test_chunked_form_is_the_recurrence(fam, lo):
    for seed in range(3):
        S0, ks, vs, a, b = _case(fam, seed, lo=lo)
        want, _ = orc.flush(fam, S0, list(zip(ks, vs, a, b)))
        got = chunked_flush(fam, S0, ks, vs, a, b)
        assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


def test_chunked_form_catches_a_dropped_pair_term():
    """Planted mistake: without the pair weights the form is wrong."""
    S0, ks, vs, a, b = _case(orc.GDN, 7)
    want, _ = orc.flush(orc.GDN, S0, list(zip(ks, vs, a, b)))
    ks2 = ks.copy()

    def no_pairs(fam, S0, ks, vs, a, b):
        W = len(ks)
        gam = [_ratio(a, t, -1) for t in range(W)]
        Y = S0.T @ ks.T
        w = np.stack([b[t] * (vs[t] - gam[t] * Y[:, t]) for t in range(W)])
        wt = np.stack([_ratio(a, W - 1, t) * w[t] for t in range(W)])
        return gam[-1] * S0 + ks.T @ wt

    assert np.abs(no_pairs(orc.GDN, S0, ks2, vs, a, b) - want).max() > 1e-3 * np.abs(want).max()


# ---------------------------------------------------------------------------
# the TF32 split plan
# ---------------------------------------------------------------------------
def _tf32(x):
    x = np.asarray(x, np.float32)
    return (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32).astype(np.float64)


def _split_mm(A, B, exact_a=False, exact_b=False, third=True):
    """fp32 operands as hi + lo; TF32 products, fp64 sums rounded to fp32.
    hi*hi + lo*hi + hi*lo, skipping the lo terms of an operand exact in TF32."""
    A = np.asarray(A, np.float32).astype(np.float64)
    B = np.asarray(B, np.float32).astype(np.float64)
    Ah, Bh = _tf32(A), _tf32(B)
    Al, Bl = A - Ah, B - Bh
    out = Ah @ Bh
    if not exact_a:
        out = out + _tf32(Al) @ Bh
    if not exact_b and third:
        out = out + Ah @ _tf32(Bl)
    return out.astype(np.float32).astype(np.float64)


def _bf16(x):
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("fam", [orc.GDN, orc.KDA])
def test_split_products_meet_the_parity_bar(fam):
    """With bf16 keys, values and queries and an fp32 basis: the flushed state,
    the exact output S_W^T q and the sketch S_W^T Omega from split TF32 products
    are within 1e-5 of the fp64 reference (the bar is 1e-4)."""
    K, V, r = 128, 128, 9
    rng = np.random.default_rng(3)
    P = np.linalg.qr(rng.standard_normal((K, r)))[0].astype(np.float32).astype(np.float64)
    worst = {"S": 0.0, "o": 0.0, "U": 0.0}
    for seed in range(3):
        S0, ks, vs, a, b = _case(fam, 10 + seed, K=K, V=V, lo=1e-2)
        S0 = S0.astype(np.float32).astype(np.float64)
        ks, vs = _bf16(ks), _bf16(vs)
        a = a.astype(np.float32).astype(np.float64)
        b = b.astype(np.float32).astype(np.float64)
        q = _bf16(rng.standard_normal(K) / np.sqrt(K))
        want, o_want = orc.flush(fam, S0, list(zip(ks, vs, a, b)), q)
        SW = chunked_flush(fam, S0, ks, vs, a, b, mm=_split_mm)
        o = _split_mm(SW.T, q[:, None], exact_b=True)[:, 0]
        U = _split_mm(SW.T, P)
        U_want = orc.sketch(want, P)
        for key, g, x in (("S", SW, want), ("o", o, o_want), ("U", U, U_want)):
            worst[key] = max(worst[key], np.abs(g - x).max() / np.abs(x).max())
    assert max(worst.values()) < 1e-5, worst


def test_two_products_are_not_enough_for_the_read_out():
    """The fp32 basis is not exact in TF32: without its lo product the sketch
    misses the bar."""
    K, V, r = 128, 128, 9
    rng = np.random.default_rng(4)
    P = np.linalg.qr(rng.standard_normal((K, r)))[0].astype(np.float32).astype(np.float64)
    S = (rng.standard_normal((K, V)) * np.sqrt(0.1)).astype(np.float32).astype(np.float64)
    U = _split_mm(S.T, P, third=False)
    want = orc.sketch(S, P)
    assert np.abs(U - want).max() / np.abs(want).max() > 1e-4
