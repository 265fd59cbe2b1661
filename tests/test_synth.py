"""The seeded input generator (ssm_decode_b200/synth.py) against the recipe it
states: determinism per (workload, step), shapes and storage formats, and the
distributions of each family's per-step inputs.  CPU only; these check the
inputs both the oracle and the library are fed, not the method.
"""
import numpy as np
import pytest

from ssm_decode_b200 import synth


def _small(name, **kw):
    return synth.shrink(synth.WORKLOADS[name], **kw)


def test_same_step_same_inputs_and_steps_differ():
    wl = _small("gdn_b256", batch=4, heads=3)
    st = synth.static_inputs(wl)
    a, b = synth.step_inputs(wl, st, 5), synth.step_inputs(wl, st, 5)
    for key in a:
        assert np.array_equal(a[key], b[key])
    c = synth.step_inputs(wl, st, 6)
    assert not np.array_equal(a["k"], c["k"])
    # the static tensors are regenerated identically too
    st2 = synth.static_inputs(wl)
    assert np.array_equal(st.state, st2.state) and np.array_equal(st.basis, st2.basis)


@pytest.mark.parametrize("name", ["mamba2_b320", "gdn_b256", "kda_b256"])
def test_shapes_and_storage_formats(name):
    wl = _small(name, batch=3)
    st = synth.static_inputs(wl)
    inp = synth.step_inputs(wl, st, 0)
    B, H, K, V = wl.batch, wl.heads, wl.dk, wl.dv
    assert inp["q"].shape == (B, H, K) and inp["q"].dtype == np.uint16
    assert inp["k"].shape == (B, H, K) and inp["k"].dtype == np.uint16
    assert inp["v"].shape == (B, H, V) and inp["v"].dtype == np.uint16
    assert inp["gate"].dtype == np.float32 and inp["beta"].dtype == np.float32
    assert inp["gate"].shape == ((B, H, K) if wl.family == synth.KDA else (B, H))
    assert st.state.shape == (B, H, K, V) and st.state.dtype == np.float32
    assert st.offsets[0] == 0 and st.offsets[-1] == len(st.basis) == st.ranks.sum()


def test_state_is_centred_with_variance_one_tenth():
    wl = _small("gdn_b256", batch=8)
    s = synth.static_inputs(wl).state.astype(np.float64)
    n = s.size                                           # 8 * 32 * 128 * 128 draws
    assert abs(s.mean()) < 5 * np.sqrt(0.1 / n)
    assert abs(s.var() - 0.1) < 5 * 0.1 * np.sqrt(2.0 / n)


def test_mamba2_step_distributions():
    wl = _small("mamba2_b320", batch=64, structured_q=False)
    st = synth.static_inputs(wl, with_state=False)
    assert np.all(st.A < 0) and np.all(st.A >= -np.exp(2.0)) and np.all(st.A <= -1.0)
    inp = synth.step_inputs(wl, st, 3)
    dt = inp["gate"].astype(np.float64)
    assert np.all(dt > 0) and np.all(inp["beta"] == 0)
    # dt = softplus(x), x ~ N(-2, 1): log(exp(dt) - 1) recovers x
    x = np.log(np.expm1(dt))
    assert abs(x.mean() + 2.0) < 0.05 and abs(x.std() - 1.0) < 0.05
    k = synth.bf16_bits_to_f32(inp["k"]).astype(np.float64)
    v = synth.bf16_bits_to_f32(inp["v"]).astype(np.float64)
    assert abs(k.var() * wl.dk - 1.0) < 0.03 and abs(v.var() - 1.0) < 0.03


@pytest.mark.parametrize("name", ["gdn_b256", "kda_b256"])
def test_delta_rule_step_distributions(name):
    wl = _small(name, batch=32)
    st = synth.static_inputs(wl, with_state=False)
    inp = synth.step_inputs(wl, st, 2)
    a = inp["gate"].astype(np.float64)
    b = inp["beta"].astype(np.float64)
    assert np.all((a > 0) & (a < 1)) and np.all((b > 0) & (b < 1))
    # a = exp(-softplus(x)) and beta = sigmoid(y), x, y ~ N(0, 1)
    x = np.log(np.expm1(-np.log(a)))
    y = np.log(b / (1 - b))
    for z in (x, y):
        assert abs(z.mean()) < 0.05 and abs(z.std() - 1.0) < 0.05
    # q and k are unit vectors up to bf16 rounding of each entry
    for key in ("q", "k"):
        nrm = np.linalg.norm(synth.bf16_bits_to_f32(inp[key]).astype(np.float64), axis=-1)
        assert np.all(np.abs(nrm - 1.0) < 2 ** -7)


def test_structured_queries_concentrate_in_the_basis():
    """q = G z + 0.1 n with G = Q diag(0.7^i): the query covariance has
    eigenvalues 0.49^i + 0.01, so the span of the top r eigenvectors (the
    basis rows) holds (sum_{i<r} 0.49^i + 0.01 r) / (sum_i 0.49^i + 0.01 dk)
    of the energy in expectation, far above the r / dk of a random subspace."""
    wl = _small("mamba2_b320", batch=256, heads=4)
    st = synth.static_inputs(wl, with_state=False)
    q = synth.bf16_bits_to_f32(synth.step_inputs(wl, st, 0)["q"]).astype(np.float64)
    lam = 0.49 ** np.arange(wl.dk) + 0.01
    for h in range(wl.heads):
        P = st.basis[st.offsets[h]:st.offsets[h + 1]].astype(np.float64)     # [r, K]
        r = len(P)
        share = np.sum((q[:, h] @ P.T) ** 2) / np.sum(q[:, h] ** 2)
        expected = lam[:r].sum() / lam.sum()
        assert abs(share - expected) < 0.05, (h, r, share, expected)
        assert share > 2.5 * r / wl.dk
