"""Randomised host checks of ss_create / ss_buffer_sizes / ss_traffic_bytes
(no GPU needed: none of them launches anything).

For arbitrary configurations, valid or not, the library must return a status
and never crash.  Every configuration that breaks a documented rule (family,
batch, heads <= 512, dk and dv in {64, 128}, 1 <= W <= 32, sketch dtype, ranks
in 0..dk, dense heads at rank dk, coefficient mode and ridge, batch * heads
<= 2^30) is refused; the configurations the header promises (fixed map, every
rank up to 64 at W <= 16 and up to 32 at W <= 32) are accepted; and an accepted
plan's buffer sizes equal the layouts the header documents, computed here from
the shapes alone.
"""
import ctypes

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import HealthCheck, event, given, settings
from hypothesis import strategies as st

from ssm_decode_b200 import binding as B
from ssm_decode_b200 import build


@pytest.fixture(scope="module")
def L():
    build.build()
    return B.lib()


def _create(L, family, batch, heads, dk, dv, window, ranks, dtype, coef_mode, ridge, dense):
    n = max(heads, 1)
    rk = (ctypes.c_int32 * n)(*(ranks + [0] * n)[:n])
    dn = None if dense is None else (ctypes.c_uint8 * n)(*(dense + [0] * n)[:n])
    cfg = B.ss_config(family, batch, heads, dk, dv, window, ctypes.cast(rk, ctypes.POINTER(ctypes.c_int32)),
                      dtype, coef_mode, ridge,
                      None if dn is None else ctypes.cast(dn, ctypes.POINTER(ctypes.c_uint8)))
    h = ctypes.c_void_p()
    status = L.ss_create(ctypes.byref(cfg), ctypes.byref(h))
    return status, h


def _map_fits(K, V, r):
    free = K * V - r * (V + 4)
    return r <= V and free >= (V // 16) * K and free >= r * r


def _lrd_fits(K, V, r):
    """The low-rank-plus-diagonal map's scratch: energies, pivots, 4 pivot
    columns, the diagonal, per-warp partials, P^T L and the Gram matrix."""
    return r <= K and V + 16 + 4 * K + K + (V // 16) * K + 4 * r + r * r <= K * V


def _breaks_a_rule(family, batch, heads, dk, dv, window, ranks, dtype, coef_mode, ridge, dense):
    if family not in (0, 1, 2) or batch < 1 or not 1 <= heads <= 512:
        return True
    if dk not in (64, 128) or dv not in (64, 128) or not 1 <= window <= 32:
        return True
    if dtype not in (0, 1) or coef_mode not in (0, 1, 2):
        return True
    if coef_mode in (1, 2) and not (ridge >= 0 and ridge < 3.0e38):
        return True
    if batch * heads > 2 ** 30:
        return True
    for h in range(heads):
        r = ranks[h]
        d = dense is not None and dense[h]
        if not 0 <= r <= dk or (d and r != dk):
            return True
        if coef_mode == 1 and not d and not _map_fits(dk, dv, r):
            return True
        if coef_mode == 2 and not d and not _lrd_fits(dk, dv, r):
            return True
    return False


def _promised(family, heads, window, ranks, coef_mode, dense):
    rmax = max(ranks[:heads])
    return coef_mode == 0 and dense is None and ((window <= 16 and rmax <= 64) or rmax <= 32)


configs = st.fixed_dictionaries({
    "family": st.sampled_from([0, 1, 2]),
    "batch": st.one_of(st.integers(1, 600), st.sampled_from([1 << 16, 1 << 21])),
    "heads": st.one_of(st.integers(1, 40), st.sampled_from([128, 512])),
    "dk": st.sampled_from([64, 128]),
    "dv": st.sampled_from([64, 128]),
    "window": st.integers(1, 32),
    "dtype": st.sampled_from([0, 1]),
    "coef_mode": st.sampled_from([0, 0, 1, 2]),
    "ridge": st.sampled_from([0.0, 0.01, 1.0]),
    "seed": st.integers(0, 2 ** 32 - 1),
    "with_dense": st.booleans(),
    # at most one rule broken per example, in about half of them
    "break": st.sampled_from([None] * 12 + ["family", "batch", "batch_heads", "heads", "dk", "dv", "window",
                                            "dtype", "coef_mode", "ridge", "rank", "dense_rank"]),
})

_BAD = {"family": [3, -1], "batch": [0, -3], "heads": [0, 513], "dk": [32, 256], "dv": [96, 32],
        "window": [0, 33], "dtype": [2, -1], "coef_mode": [3, -1]}


@settings(max_examples=400, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(c=configs)
def test_random_configs(L, c):
    import random
    c = dict(c)
    rnd = random.Random(c["seed"])
    brk = c["break"]
    if brk in _BAD:
        c[brk] = rnd.choice(_BAD[brk])
    if brk == "batch_heads":
        c["heads"], c["batch"] = 512, (1 << 21) + 1               # batch * heads just above 2^30
    if brk == "ridge":
        c["coef_mode"], c["ridge"] = rnd.choice([1, 2]), rnd.choice([-1.0, float("inf"), float("nan")])
    heads, dk = c["heads"], c["dk"]
    n = max(heads, 1)
    hi = dk if dk in (64, 128) else 128
    cap = rnd.choice([8, 16, 32, 64, hi])                          # largest rank in this plan
    ranks = [rnd.randint(0, min(cap, hi)) for _ in range(n)]
    dense = None
    if c["with_dense"]:
        dense = [1 if rnd.random() < 0.15 else 0 for _ in range(n)]
        ranks = [dk if d else r for d, r in zip(dense, ranks)]
    if brk == "rank":
        ranks[rnd.randrange(n)] = rnd.choice([-1, hi + 1])
    if brk == "dense_rank":
        dense = dense or [0] * n
        i = rnd.randrange(n)
        dense[i], ranks[i] = 1, rnd.randint(0, hi - 1)
    args = (c["family"], c["batch"], heads, dk, c["dv"], c["window"], ranks, c["dtype"], c["coef_mode"],
            c["ridge"], dense)
    status, h = _create(L, *args)
    try:
        if _breaks_a_rule(*args):
            event("refused: breaks a rule")
            assert status != B.SS_OK, args
            assert h.value is None
            assert L.ss_last_error_string().decode()
            return
        if _promised(c["family"], heads, c["window"], ranks, c["coef_mode"], dense):
            assert status == B.SS_OK, (args, L.ss_last_error_string().decode())
        if status != B.SS_OK:
            # the only other refusal: the launch would not fit in shared memory
            assert status == B.SS_ERR_UNSUPPORTED
            assert "shared memory" in L.ss_last_error_string().decode()
            event("refused: shared memory")
            return
        event("accepted")
        s = B.ss_sizes()
        assert L.ss_buffer_sizes(h, ctypes.byref(s)) == B.SS_OK
        Bt, H, K, V, W = c["batch"], heads, dk, c["dv"], c["window"]
        fam, esz = c["family"], 2 if c["dtype"] == B.SS_BF16 else 4
        R = sum(ranks[:H])
        Wg = (W + 3) // 4 * 4
        assert s.total_rank == R
        assert s.state == Bt * H * K * V * 4
        assert s.ring_k == Bt * H * W * K * 2 and s.ring_v == Bt * H * W * V * 2
        assert s.ring_gate == (Bt * H * W * K if fam == B.SS_KDA else Bt * H * Wg) * 4
        assert s.ring_beta == (0 if fam == B.SS_MAMBA2 else Bt * H * Wg * 4)
        assert s.sketch == Bt * R * V * esz
        assert s.basis == R * K * 4 and s.coef == R * K * 4
        assert s.A == (H * 4 if fam == B.SS_MAMBA2 else 0)
        assert s.q == Bt * H * K * 2 and s.k == Bt * H * K * 2 and s.v == Bt * H * V * 2
        assert s.gate == (Bt * H * K if fam == B.SS_KDA else Bt * H) * 4
        assert s.beta == (0 if fam == B.SS_MAMBA2 else Bt * H * 4)
        assert s.out == Bt * H * V * 4
        assert s.coef_state == (Bt * R * K * esz if c["coef_mode"] in (B.SS_COEF_STATE, B.SS_COEF_LRD) else 0)
        assert s.gate_stride == (W * K if fam == B.SS_KDA else Wg)
        # traffic: defined for every phase the schedule allows, linear in the phase
        t = B.ss_traffic()
        reads = []
        for tau in range(W - 1):
            assert L.ss_traffic_bytes(h, B.SS_OP_DECODE, tau, ctypes.byref(t)) == B.SS_OK
            assert t.read_bytes > 0 and t.write_bytes > 0 and t.paper_read_bytes >= 0
            reads.append(t.read_bytes)
        if len(reads) >= 3:
            steps = {round(b - a, 3) for a, b in zip(reads, reads[1:])}
            assert len(steps) == 1 and min(steps) > 0
        assert L.ss_traffic_bytes(h, B.SS_OP_DECODE, W - 1, ctypes.byref(t)) != B.SS_OK
        assert L.ss_traffic_bytes(h, B.SS_OP_FLUSH, 0, ctypes.byref(t)) == B.SS_OK
        assert t.read_bytes >= s.state and t.write_bytes >= s.state
    finally:
        if h.value:
            L.ss_destroy(h)
