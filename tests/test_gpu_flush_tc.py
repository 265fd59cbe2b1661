"""GPU parity of the tensor-core flush against the fp64 oracle (needs a B200).

GDN and KDA flushes with dv = 128, dk = 64 or 128, at most 16 buffered
updates and at most 32 read-out columns per head run on the fifth-generation
tensor cores (tf32 operands split into hi and lo halves, GDN's Gram products in
bf16 parts).  These cases walk that kernel's edges: every window length up to
16 (the update count sets the recursion's size and the MN-major key blocks),
ranks from 0 to 31 with the token's column (read-out widths 16 and 32),
both sketch dtypes, the end-of-sequence flush without a token, the identity
transition bit for bit, and more heads than SMs, so that each persistent CTA
pipelines several heads through its barriers.
"""
import numpy as np
import pytest

from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from tests.parity_util import TOL, Pair
from tests.test_gpu_parity import FAM, run, small

pytestmark = pytest.mark.gpu


def with_ranks(wl, ranks, seed):
    """Static inputs whose heads have the given ranks (orthonormal bases)."""
    st = synth.static_inputs(wl)
    ranks = np.asarray(ranks, np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    basis = np.concatenate([np.linalg.qr(rng.standard_normal((wl.dk, wl.dk)))[0][:, :r].T
                            for r in ranks]).astype(np.float32)
    st.ranks, st.offsets, st.basis, st.coef = ranks, offs, basis, basis.copy()
    return st


@pytest.mark.parametrize("window", [1, 2, 3, 5, 9, 16])
@pytest.mark.parametrize("dk", [128, 64])
@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_windows(cuda_ok, family, dk, window):
    wl = small(FAM[family], dk, 128, batch=2, heads=3, window=window, seed=2000 + dk + window)
    w = run(Pair(wl), 2 * window + 3)
    assert w["state"] <= TOL and w["sketched"] <= TOL


@pytest.mark.parametrize("sketch", ["f32", "bf16"])
@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_ranks_up_to_read_out_width(cuda_ok, family, sketch):
    """Ranks 0, 1, 15, 16 and 31: read-out widths 1 to 32 with the token."""
    wl = small(FAM[family], 128, 128, heads=5, seed=2100)
    st = with_ranks(wl, [0, 1, 15, 16, 31], seed=21)
    dt = B.SS_BF16 if sketch == "bf16" else B.SS_F32
    run(Pair(wl, st=st, sketch_dtype=dt), 2 * wl.window + 2)


@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_narrow_read_out(cuda_ok, family):
    """Every rank at most 15: the 16-column read-out layout."""
    wl = small(FAM[family], 64, 128, heads=4, seed=2200)
    st = with_ranks(wl, [3, 15, 0, 8], seed=22)
    run(Pair(wl, st=st), wl.window + 4)


@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_flush_without_token(cuda_ok, family):
    """End of sequence: the tau buffered updates and no token (no output column)."""
    wl = small(FAM[family], 128, 128, seed=2300)
    p = Pair(wl)
    p.prime()
    for t in range(7):
        p.step(synth.step_inputs(wl, p.st, t))
    p.layer.flush(None)
    p.sess.flush(None)
    p.check_state()
    p.check_sketch()
    assert p.layer.phase == 0


@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_identity_bit_exact(cuda_ok, family):
    """Unit decays and zero update strengths: the state is unchanged bit for bit."""
    import torch
    wl = small(FAM[family], 128, 128, seed=2400)
    p = Pair(wl)
    before = p.layer.state.clone()
    p.layer.prime()
    assert torch.equal(p.layer.state, before)
    for t in range(wl.window):
        inp = synth.step_inputs(wl, p.st, t)
        inp["gate"][:] = 1.0
        inp["beta"][:] = 0.0
        p.layer.step(p.layer.token(inp))
    torch.cuda.synchronize()
    assert p.layer.phase == 0
    assert torch.equal(p.layer.state, before)


@pytest.mark.parametrize("family", ["gdn", "kda"])
def test_tc_heads_beyond_one_wave(cuda_ok, family):
    """More heads than SMs: each CTA carries several heads through its pipeline."""
    wl = small(FAM[family], 128, 128, batch=64, heads=5, window=16, seed=2500)
    w = run(Pair(wl), 2 * wl.window + 1)
    assert w["state"] <= TOL
