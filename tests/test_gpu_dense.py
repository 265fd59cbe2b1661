"""GPU parity of dense-fallback heads (paper App. D: at non-flush steps such
heads read a BF16 copy of their state instead of a sketch).

A dense head has rank dk; every flush with a sketch writes its state into its
sketch rows (row k = S[k][:], in the sketch dtype) and its non-flush read is
S0^T q~ + (buffered term) from that copy.  The oracle session models it as
the identity basis and map (u_k = S0^T e_k = row k of S0, c = q~), so the
read is exact up to the copy's rounding.  Dense and sketched heads are mixed
in every case, with ragged ranks on the sketched ones.
"""
import numpy as np
import pytest

from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from tests.parity_util import TOL, Pair, to_np

pytestmark = pytest.mark.gpu

FAM = {"mamba2": synth.MAMBA2, "gdn": synth.GDN, "kda": synth.KDA}


def case(family, dk, dv, window=6, heads=4, batch=3, dense=(1, 0, 0, 1), seed=2300):
    """Static inputs with the dense heads' ranks raised to dk (their basis and
    map rows are filler the library must not read)."""
    wl = synth.Workload(f"dense_{family}", FAM[family], batch, heads, dk, dv, window, 0, 8, seed)
    st = synth.static_inputs(wl)
    dense = np.asarray(dense, bool)
    ranks = np.where(dense, dk, st.ranks).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    rows = []
    for h in range(heads):
        if dense[h]:
            rows.append(np.full((dk, dk), np.nan, np.float32))      # never read
        else:
            rows.append(st.basis[st.offsets[h]:st.offsets[h + 1]])
    basis = np.concatenate(rows).astype(np.float32)
    st.ranks, st.offsets, st.basis, st.coef = ranks, offs, basis, basis.copy()
    return wl, st, dense


def run(pair, steps):
    pair.prime()
    for t in range(steps):
        pair.step(synth.step_inputs(pair.wl, pair.st, t))
    return pair


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128)])
@pytest.mark.parametrize("sketch_dtype", [B.SS_F32, B.SS_BF16])
def test_dense_heads_read_their_state_copy(cuda_ok, family, dk, dv, sketch_dtype):
    wl, st, dense = case(family, dk, dv, seed=2300 + dk)
    p = run(Pair(wl, st=st, sketch_dtype=sketch_dtype, dense=dense), 2 * wl.window + 2)
    # the copy itself: row k of a dense head's sketch rows is S[k][:]
    import torch
    g = to_np(p.layer.sketch)
    for h in np.flatnonzero(dense):
        lo = st.offsets[h]
        want = p.layer.state[:, h]
        want = to_np(want if sketch_dtype == B.SS_F32 else want.to(torch.bfloat16))
        assert np.array_equal(g[:, lo:lo + dk], want), f"head {h}: the state copy is not the state"


@pytest.mark.parametrize("family", ["mamba2", "gdn"])
def test_dense_heads_with_state_map(cuda_ok, family):
    """Sketched heads with the state-dependent map beside dense heads."""
    wl, st, dense = case(family, 128, 128, seed=2400)
    run(Pair(wl, st=st, state_map=True, rho=0.1, dense=dense), 2 * wl.window + 1)


def test_all_heads_dense(cuda_ok):
    wl, st, dense = case("kda", 64, 64, heads=3, dense=(1, 1, 1), seed=2500)
    run(Pair(wl, st=st, sketch_dtype=B.SS_BF16, dense=dense), wl.window + 2)


def test_dense_heads_full_size_sampled(cuda_ok):
    """The GDN batch-256 workload with every fourth head dense, sampled."""
    wl = synth.WORKLOADS["gdn_b256"]
    st = synth.static_inputs(wl)
    dense = (np.arange(wl.heads) % 4) == 0
    ranks = np.where(dense, wl.dk, st.ranks).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rows = [np.eye(wl.dk, dtype=np.float32) if dense[h] else st.basis[st.offsets[h]:st.offsets[h + 1]]
            for h in range(wl.heads)]
    st.ranks, st.offsets = ranks, offs
    st.basis = np.concatenate(rows).astype(np.float32)
    st.coef = st.basis.copy()
    p = Pair(wl, st=st, sketch_dtype=B.SS_BF16, sel=[0, 128, 255], dense=dense)
    run(p, wl.window + 1)


def test_flush_with_failed_dense_copy_needs_prime(cuda_ok):
    """The flush is queued but the dense heads' copy launch is refused (the
    host-side testing hook stands in for the runtime's refusal): the call
    returns SS_ERR_CUDA, the window has been applied exactly once, and the
    plan sits at phase 0 with no valid sketch, so reads are refused until
    ss_prime rebuilds the sketch and the copies."""
    import torch
    wl, st, dense = case("gdn", 128, 64, window=4, seed=2600)
    p = Pair(wl, st=st, dense=dense)
    p.prime()
    for t in range(wl.window - 1):
        p.step(synth.step_inputs(wl, st, t))
    inp = synth.step_inputs(wl, st, wl.window - 1)
    tok = p.layer.token(inp)
    B.ss_debug_fail_launch(p.layer.plan, 2)            # launch 1: the flush; launch 2: the copies
    with pytest.raises(B.SSError) as err:
        p.layer.flush(tok)
    assert "injected" in str(err.value)
    assert B.ss_get_phase(p.layer.plan) == (0, 0)
    torch.cuda.synchronize()
    o = p.sess.flush(inp)                               # the oracle's flush of the same window
    p.check_state()
    from tests.parity_util import vec_relerr
    assert vec_relerr(p.out(), o) <= TOL
    with pytest.raises(B.SSError):                      # no sketch: a read is a schedule error
        p.layer.decode(p.layer.token(synth.step_inputs(wl, st, wl.window)))
    p.layer.prime()                                     # the hook has fired: this runs
    p.sess.prime()
    p.check_sketch()
    for t in range(wl.window, wl.window + 3):
        p.step(synth.step_inputs(wl, st, t))
