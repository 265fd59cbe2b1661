"""GPU parity of libsketchssm.so against the fp64 oracle (needs a B200).

Every call goes through the C ABI (ctypes).  Sizes are small enough for the
oracle to finish in seconds but span several column tiles, both CTA packings
(dv = 64: two heads per CTA, with a ragged last CTA) and ragged ranks
(including 0 and 1); full-size workloads are compared on sampled sequences.
"""
import numpy as np
import pytest

from oracle import sketchssm_oracle as orc
from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from tests.parity_util import TOL, Pair, head_relerr, to_np, vec_relerr

pytestmark = pytest.mark.gpu

FAM = {"mamba2": synth.MAMBA2, "gdn": synth.GDN, "kda": synth.KDA}


def small(family, dk=128, dv=128, batch=3, heads=5, window=16, steps=20, mean_rank=8, seed=77):
    return synth.Workload(f"small_{family}", family, batch, heads, dk, dv, window, steps, mean_rank,
                          seed)


def run(pair, steps, t0=0):
    pair.prime()
    for t in range(t0, t0 + steps):
        pair.step(synth.step_inputs(pair.wl, pair.st, t))
    return pair.worst


# ---------------------------------------------------------------------------
def test_mamba2_b4_full_session(cuda_ok):
    """The small Mamba-2 case in full: 64 steps (4 windows), every output."""
    wl = synth.WORKLOADS["mamba2_b4"]
    w = run(Pair(wl), wl.steps)
    assert w["out"] <= TOL and w["sketched"] <= TOL and w["state"] <= TOL


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_families_and_shapes(cuda_ok, family, dk, dv):
    wl = small(FAM[family], dk, dv, seed=100 + dk + dv)
    run(Pair(wl), 20)


@pytest.mark.parametrize("window", [1, 2, 3, 5, 32])
@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_windows(cuda_ok, family, window):
    wl = small(FAM[family], 128, 64, batch=2, heads=3, window=window, seed=300 + window)
    run(Pair(wl), 2 * window + 3)


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_bf16_sketch(cuda_ok, family):
    wl = small(FAM[family], 128, 128 if family != "mamba2" else 64, seed=400)
    run(Pair(wl, sketch_dtype=B.SS_BF16), 20)


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_ragged_ranks_with_zero_and_one(cuda_ok, family):
    wl = small(FAM[family], 128, 64, heads=4, seed=500)
    st = synth.static_inputs(wl)
    ranks = np.array([0, 1, 16, 7], np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rng = np.random.default_rng(5)
    basis = np.concatenate([np.linalg.qr(rng.standard_normal((wl.dk, wl.dk)))[0][:, :r].T
                            for r in ranks]).astype(np.float32)
    st.ranks, st.offsets, st.basis, st.coef = ranks, offs, basis, basis.copy()
    run(Pair(wl, st=st), 18)


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_standard_exact_step(cuda_ok, family, dk, dv):
    """The Standard baseline (paper App. D): every step reads and writes the
    full state; output and state against the oracle's recurrence."""
    wl = small(FAM[family], dk, dv, seed=600 + dk + dv)
    p = Pair(wl)
    for t in range(6):
        p.exact_step(synth.step_inputs(wl, p.st, t))


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_replay_window(cuda_ok, family, dk, dv):
    """The ReplaySSM baseline (GitHub page "Overview"; paper App. D): exact
    windowed reads of S0 and a flush without a sketch, over two windows and
    a part of a third."""
    wl = small(FAM[family], dk, dv, window=8, seed=700 + dk + dv)
    p = Pair(wl)
    for t in range(19):
        p.replay_step(synth.step_inputs(wl, p.st, t))


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_flush_without_token(cuda_ok, family):
    """End of sequence: flush the tau buffered updates with no new token."""
    wl = small(FAM[family], 128, 64, seed=800)
    p = Pair(wl)
    p.prime()
    for t in range(5):
        p.step(synth.step_inputs(wl, p.st, t))
    p.layer.flush(None)
    p.sess.flush(None)
    p.check_state()
    p.check_sketch()
    assert p.layer.phase == 0


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_full_rank_identity_basis_is_exact(cuda_ok, family):
    """P = I with r = dk (and C = I): sketched reads equal exact reads."""
    wl = small(FAM[family], 64, 64, batch=2, heads=3, seed=900)
    st = synth.static_inputs(wl)
    st.ranks = np.full(wl.heads, wl.dk, np.int32)
    st.offsets = (np.arange(wl.heads + 1) * wl.dk).astype(np.int32)
    st.basis = np.tile(np.eye(wl.dk, dtype=np.float32), (wl.heads, 1))
    st.coef = st.basis.copy()
    p = Pair(wl, st=st)
    p.prime()
    for t in range(wl.window + 3):
        inp = synth.step_inputs(wl, st, t)
        ph = p.layer.phase
        p.step(inp)
        if ph != wl.window - 1:
            # the sketched output equals the oracle's exact windowed read
            qt, ob = orc.effective_query(wl.family, p.sess.ring, p.sess.token(inp)[0])
            exact = orc.read(p.sess.S, qt) + ob
            assert vec_relerr(p.out(), exact) <= TOL


@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_flush_identity_bit_exact(cuda_ok, family):
    """Zero decay rate and zero update strength: the state is unchanged bit for bit."""
    import torch
    wl = small(FAM[family], 128, 64, seed=1000)
    p = Pair(wl)
    before = p.layer.state.clone()
    p.layer.prime()
    assert torch.equal(p.layer.state, before)
    for t in range(wl.window):
        inp = synth.step_inputs(wl, p.st, t)
        if family == "mamba2":
            inp["gate"][:] = 0.0                     # dt = 0: a = 1, b = 0
        else:
            inp["gate"][:] = 1.0
            inp["beta"][:] = 0.0
        p.layer.step(p.layer.token(inp))
    torch.cuda.synchronize()
    assert p.layer.phase == 0
    assert torch.equal(p.layer.state, before)


@pytest.mark.parametrize("family", ["gdn", "kda", "mamba2"])
def test_strong_decay_renormalisation(cuda_ok, family):
    """Decays small enough to force the kernel's renormalisation, and exact zeros."""
    wl = small(FAM[family], 128, 128, window=16, seed=1100)
    p = Pair(wl)
    p.prime()
    rng = np.random.default_rng(11)
    for t in range(20):
        inp = synth.step_inputs(wl, p.st, t)
        if family == "mamba2":
            inp["gate"] = (inp["gate"] * 40.0).astype(np.float32)          # exp(dt A) down to ~1e-30
        else:
            g = inp["gate"]
            g = (g * (10.0 ** rng.uniform(-9, 0, g.shape))).astype(np.float32)
            g[rng.uniform(size=g.shape) < 0.05] = 0.0                      # exact resets
            inp["gate"] = g
        p.step(inp)


def test_checkpoint_resume_is_bit_identical(cuda_ok):
    import torch
    wl = small(synth.GDN, 128, 128, seed=1200)
    p = Pair(wl)
    p.layer.prime()
    L = p.layer
    for t in range(5):
        L.step(L.token(synth.step_inputs(wl, p.st, t)))
    names = ["state", "ring_k", "ring_v", "ring_gate", "ring_beta", "sketch"]
    snap = {n: getattr(L, n).clone() for n in names}
    phase, valid = B.ss_get_phase(L.plan)
    outs = []
    for t in range(5, 25):
        L.step(L.token(synth.step_inputs(wl, p.st, t)))
        outs.append(L.out.clone())
    for n in names:
        getattr(L, n).copy_(snap[n])
    B.ss_set_phase(L.plan, phase, valid)
    for i, t in enumerate(range(5, 25)):
        L.step(L.token(synth.step_inputs(wl, p.st, t)))
        assert torch.equal(L.out, outs[i])


def test_launch_count(cuda_ok):
    wl = small(synth.MAMBA2, 64, 64, seed=1300)
    p = Pair(wl)
    n0 = B.ss_launch_count()
    p.layer.prime()
    p.layer.step(p.layer.token(synth.step_inputs(wl, p.st, 0)))
    assert B.ss_launch_count() == n0 + 2


def test_max_heads_and_window(cuda_ok):
    """Largest supported head count and window, rank up to 32."""
    wl = synth.Workload("maxh", synth.GDN, 1, 512, 128, 128, 32, 34, 16, 1400)
    run(Pair(wl), 34)


# ---------------------------------------------------------------------------
# full-size workloads, compared on sampled sequences
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["mamba2_b320", "gdn_b256", "kda_b256"])
@pytest.mark.parametrize("sketch", ["f32", "bf16"])
def test_full_size_sampled(cuda_ok, name, sketch):
    wl = synth.WORKLOADS[name]
    sel = [0, wl.batch // 2 + 1, wl.batch - 1]
    dt = B.SS_F32 if sketch == "f32" else B.SS_BF16
    p = Pair(wl, sketch_dtype=dt, sel=sel)
    p.prime()
    # two full windows and two steps of a third: the second window's decodes
    # read a sketch written by a full-size flush, and the second flush's state
    # and sketch are compared again
    for t in range(2 * wl.window + 2):
        p.step(synth.step_inputs(wl, p.st, t), ring=False)
    # properties that hold at any size: all outputs finite, ring slots hold the inputs
    g = to_np(p.layer.out)
    assert np.isfinite(g).all()
    inp = synth.step_inputs(wl, p.st, 2 * wl.window + 1)
    assert np.array_equal(to_np(p.layer.ring_k)[:, :, 1], inp["k"])
    assert p.worst["state"] <= TOL and p.worst["out"] <= TOL


@pytest.mark.parametrize("batch,window,mean_rank", [(1, 4, 4), (32, 32, 16), (1024, 8, 8)])
def test_sweep_points_sampled(cuda_ok, batch, window, mean_rank):
    wl = synth.sweep_workload(batch, window, mean_rank)
    sel = sorted({0, batch // 2, batch - 1})
    p = Pair(wl, sketch_dtype=B.SS_BF16, sel=sel)
    p.prime()
    for t in range(window + 2):
        p.step(synth.step_inputs(wl, p.st, t), ring=False)


@pytest.mark.parametrize("call", ["decode", "replay", "flush"])
def test_bounded_wait_reports_timeout(cuda_ok, call):
    """A launch whose bulk copies deliver fewer bytes than one CTA expects: that
    CTA's bounded wait runs out, it sets SS_DEVICE_TIMEOUT in the status word
    and returns; the context stays usable and later launches are clean."""
    import torch
    wl = small(synth.GDN, 128, 128, batch=4, heads=3, seed=1500)
    p = Pair(wl)
    p.layer.prime()
    torch.cuda.synchronize()
    assert int(p.layer.status[0]) == 0
    B.ss_debug_stall_next_copy(p.layer.plan, True)
    tok = p.layer.token(synth.step_inputs(wl, p.st, 0))
    if call == "decode":
        p.layer.decode(tok)
    elif call == "replay":
        B.ss_replay_step(p.layer.plan, p.layer.bufs(False), p.layer.io(tok))
    else:
        p.layer.flush(None)                      # end-of-sequence flush of an empty window
    torch.cuda.synchronize()
    assert int(p.layer.status[0]) & B.SS_DEVICE_TIMEOUT
    # the context is still usable: a fresh session runs clean and matches the oracle
    q = Pair(wl)
    run(q, 6)
    torch.cuda.synchronize()
    assert int(q.layer.status[0]) == 0
