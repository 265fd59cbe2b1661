"""Mixed-phase batches on the GPU: every sequence at its own window position.

One ss_step_mixed call decodes the sequences whose window still has room and
flushes the ones at position W-1 (SketchSSM project page, "Per step": the
flush/non-flush choice is made per sequence).  Each sequence is checked
against its own fp64 oracle Session, which follows the single-sequence
schedule of the paper (§3.2 non-flush reads, §4.1 flush).  The rings are
filled to the starting positions by writing the raw inputs into the ring
slots, which is the layout include/sketchssm.h fixes for ss_step_io's fields.
"""
import numpy as np
import pytest

from oracle import sketchssm_oracle as orc
from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from ssm_decode_b200.layer import DecodeLayer
from tests.parity_util import TOL, head_relerr, to_np, vec_relerr

pytestmark = pytest.mark.gpu

FAM = {"mamba2": synth.MAMBA2, "gdn": synth.GDN, "kda": synth.KDA}


def _one(inp, b):
    return {k: v[b:b + 1] for k, v in inp.items()}


def _put_ring(layer, inp, b, slot):
    """Buffer sequence b's raw token at ring slot `slot`, bit for bit."""
    import torch
    dev = layer.device
    layer.ring_k[b, :, slot] = torch.from_numpy(inp["k"][b].view(np.int16)).to(dev)
    layer.ring_v[b, :, slot] = torch.from_numpy(inp["v"][b].view(np.int16)).to(dev)
    layer.ring_gate[b, :, slot] = torch.from_numpy(inp["gate"][b]).to(dev)   # [H] or KDA's [H, dk]
    if layer.family != B.SS_MAMBA2:
        layer.ring_beta[b, :, slot] = torch.from_numpy(inp["beta"][b]).to(dev)


def _setup(family, window, batch, fills, seed, dk=128, dv=64, heads=3):
    import torch
    wl = synth.Workload(f"mixed_{family}", FAM[family], batch, heads, dk, dv, window, 0, 8, seed)
    st = synth.static_inputs(wl)
    layer = DecodeLayer(wl.family, batch, heads, dk, dv, window, st.ranks)
    layer.load(st.state, st.basis, st.coef, st.A)
    sess = [orc.Session(wl.family, st.state[b:b + 1], window, st.A, st.basis, st.coef, st.offsets)
            for b in range(batch)]
    layer.prime()
    for s in sess:
        s.prime()
    # Bring sequence b to fill fills[b]: its first fills[b] buffered tokens.
    for j in range(max(fills) if len(fills) else 0):
        inp = synth.step_inputs(wl, st, 500 + j)
        for b in range(batch):
            if j < fills[b]:
                _put_ring(layer, inp, b, j)
                sess[b].decode(_one(inp, b))
    torch.cuda.synchronize()
    return wl, st, layer, sess


def _check_step(layer, sess, inp, fill, wl):
    """Compare one mixed step's outputs (and, for flushed sequences, state and
    sketch) with each sequence's oracle."""
    g = to_np(layer.out)
    S = to_np(layer.state)
    U = to_np(layer.sketch)
    for b, s in enumerate(sess):
        if fill[b] == wl.window - 1:
            o = s.flush(_one(inp, b))
            err = vec_relerr(g[b:b + 1], o)
            assert err <= TOL, f"seq {b} flush output relerr {err:.3e}"
            err = head_relerr(S[b:b + 1], s.S)
            assert err <= TOL, f"seq {b} state relerr {err:.3e}"
            ref = s.packed_sketch()
            offs = s.offsets
            for h in range(wl.heads):
                if offs[h + 1] > offs[h]:
                    err = head_relerr(U[b:b + 1, offs[h]:offs[h + 1]], ref[:, offs[h]:offs[h + 1]])
                    assert err <= TOL, f"seq {b} sketch head {h} relerr {err:.3e}"
        else:
            o_hat, _ = s.decode(_one(inp, b))
            err = vec_relerr(g[b:b + 1], o_hat)
            assert err <= TOL, f"seq {b} at fill {fill[b]}: sketched output relerr {err:.3e}"


@pytest.mark.parametrize("window", [1, 2, 5, 16])
@pytest.mark.parametrize("family", ["mamba2", "gdn", "kda"])
def test_mixed_positions_match_per_sequence_oracle(cuda_ok, family, window):
    """Every starting position 0..W-1 is present (ragged: the batch is not a
    multiple of the decode's units per warp), run for more than a window so
    each sequence flushes once or twice and decodes from a fresh sketch."""
    import torch
    batch = 11
    rng = np.random.default_rng(window)
    fills = rng.permutation(np.arange(batch) % window).astype(np.int32)
    wl, st, layer, sess = _setup(family, window, batch, fills, seed=1100 + window)
    fin = torch.from_numpy(fills).cuda()
    fout = torch.full_like(fin, -7)
    fill = fills.copy()
    for t in range(window + 4):
        inp = synth.step_inputs(wl, st, t)
        layer.step_mixed(layer.token(inp), fin, fout)
        torch.cuda.synchronize()
        _check_step(layer, sess, inp, fill, wl)
        fill = (fill + 1) % window
        assert np.array_equal(fout.cpu().numpy(), fill), "fill_out is not (fill_in + 1) mod W"
        fin, fout = fout, fin
    assert int(layer.status[0].item()) == 0
    assert layer.phase == 0


@pytest.mark.parametrize("family", ["mamba2", "gdn"])
def test_mixed_uniform_equals_scheduled_steps(cuda_ok, family):
    """All sequences at the same position: the mixed step reproduces the
    ordinary decode and flush calls bit for bit."""
    import torch
    W, batch = 4, 6
    fills = np.zeros(batch, np.int32)
    wl, st, a, _ = _setup(family, W, batch, fills, seed=1200)
    b_layer = DecodeLayer(wl.family, batch, wl.heads, wl.dk, wl.dv, W, st.ranks)
    b_layer.load(st.state, st.basis, st.coef, st.A)
    b_layer.prime()
    fin = torch.zeros(batch, dtype=torch.int32, device="cuda")
    fout = torch.empty_like(fin)
    for t in range(2 * W):
        inp = synth.step_inputs(wl, st, t)
        a.step_mixed(a.token(inp), fin, fout)
        b_layer.step(b_layer.token(inp))
        torch.cuda.synchronize()
        assert torch.equal(a.out, b_layer.out), f"step {t}: outputs differ"
        fin, fout = fout, fin
    assert torch.equal(a.state, b_layer.state)
    assert torch.equal(a.sketch, b_layer.sketch)
    assert torch.equal(a.ring_k, b_layer.ring_k)


@pytest.mark.parametrize("W", [1, 4])
def test_mixed_bad_fill_sets_status_and_skips(cuda_ok, W):
    """Fill counts outside 0..W-1 are refused on the device: the status word
    gets SS_DEVICE_BAD_FILL and those sequences are left untouched; the
    others step normally.  At W = 1 no decode kernel runs, so the flush's
    unit queue is the one that reports the bad fills."""
    import torch
    batch = 5
    fills = np.array([0, 1, 2, 3, 0], np.int32) % W
    wl, st, layer, sess = _setup("gdn", W, batch, fills, seed=1300)
    bad = fills.copy()
    bad[1], bad[4] = W, -1
    fin = torch.from_numpy(bad).cuda()
    fout = torch.full_like(fin, -7)
    layer.out.fill_(12.5)
    ring_before = layer.ring_k.clone()
    inp = synth.step_inputs(wl, st, 0)
    layer.step_mixed(layer.token(inp), fin, fout)
    torch.cuda.synchronize()
    assert int(layer.status[0].item()) == B.SS_DEVICE_BAD_FILL
    g = to_np(layer.out)
    assert (g[[1, 4]] == 12.5).all(), "a sequence with a bad fill was written"
    assert torch.equal(layer.ring_k[[1, 4]], ring_before[[1, 4]])
    assert fout[1].item() == -7 and fout[4].item() == -7
    for b in (0, 2, 3):
        if fills[b] == W - 1:
            o = sess[b].flush(_one(inp, b))
        else:
            o, _ = sess[b].decode(_one(inp, b))
        assert vec_relerr(g[b:b + 1], o) <= TOL
    layer.status.zero_()


def test_mixed_host_checks(cuda_ok):
    """Host-side refusals: aliasing fills, a missing sketch, a plan mid-window."""
    import torch
    W, batch = 4, 3
    fills = np.zeros(batch, np.int32)
    wl, st, layer, _ = _setup("mamba2", W, batch, fills, seed=1400)
    tok = layer.token(synth.step_inputs(wl, st, 0))
    f = torch.zeros(batch, dtype=torch.int32, device="cuda")
    with pytest.raises(B.SSError):
        layer.step_mixed(tok, f, f)
    g = torch.zeros_like(f)
    layer.decode(tok)                                   # plan phase 1
    with pytest.raises(B.SSError):
        layer.step_mixed(tok, f, g)


@pytest.mark.parametrize("fail_at", [1, 2])
def test_mixed_launch_failure_still_joins(cuda_ok, fail_at):
    """A mixed step whose flush (fail_at 1) or decode (fail_at 2) launch is
    refused on the host: SS_ERR_CUDA comes back, the side stream has been
    joined to the caller's stream, and whatever was queued ran to the
    oracle's values; the next mixed step on the same plan runs normally."""
    import torch
    W, batch = 4, 4
    fills = np.array([3, 1, 3, 0], np.int32)
    wl, st, layer, sess = _setup("kda", W, batch, fills, seed=1500)
    fin = torch.from_numpy(fills).cuda()
    fout = torch.full_like(fin, -7)
    layer.out.fill_(12.5)
    inp = synth.step_inputs(wl, st, 0)
    B.ss_debug_fail_launch(layer.plan, fail_at)
    with pytest.raises(B.SSError) as err:
        layer.step_mixed(layer.token(inp), fin, fout)
    assert "injected" in str(err.value)
    marker = torch.zeros(1, device="cuda")
    marker.add_(1.0)                                    # queued after the join on the caller's stream
    torch.cuda.synchronize()
    assert marker.item() == 1.0
    g = to_np(layer.out)
    flushing = [b for b in range(batch) if fills[b] == W - 1]
    decoding = [b for b in range(batch) if fills[b] != W - 1]
    if fail_at == 1:                                    # nothing ran
        assert (g == 12.5).all()
        assert (to_np(fout) == -7).all()
        return
    for b in flushing:                                  # the flush ran; the decode did not
        o = sess[b].flush(_one(inp, b))
        assert vec_relerr(g[b:b + 1], o) <= TOL
        assert head_relerr(to_np(layer.state)[b:b + 1], sess[b].S) <= TOL
        assert int(fout[b].item()) == 0
    for b in decoding:
        assert (g[b] == 12.5).all()
    # the plan is still usable: the decoding sequences step now, the flushed ones start a window
    nf = torch.from_numpy(np.where(fills == W - 1, 0, fills)).cuda().to(torch.int32)
    nout = torch.empty_like(nf)
    inp2 = synth.step_inputs(wl, st, 1)
    layer.step_mixed(layer.token(inp2), nf, nout)
    torch.cuda.synchronize()
    g2 = to_np(layer.out)
    for b in range(batch):
        o, _ = sess[b].decode(_one(inp2, b))
        assert vec_relerr(g2[b:b + 1], o) <= TOL
