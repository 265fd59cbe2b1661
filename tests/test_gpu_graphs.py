"""The decode path under CUDA graph capture, and mixed steps with dense heads.

Every library call only queues kernels on the caller's stream (the mixed
step forks its flush onto a plan-owned stream and joins it back with events),
so a window of steps can be captured once and replayed: the replay must
reproduce eager execution bit for bit.
"""
import numpy as np
import pytest

from oracle import sketchssm_oracle as orc
from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from ssm_decode_b200.layer import DecodeLayer
from tests.parity_util import TOL, to_np, vec_relerr
from tests.test_gpu_mixed import _one, _put_ring

pytestmark = pytest.mark.gpu


def _pair_of_layers(family, W=4, batch=5, heads=3, dk=128, dv=64, seed=2600, **kw):
    wl = synth.Workload(f"graph_{family}", family, batch, heads, dk, dv, W, 0, 8, seed)
    st = synth.static_inputs(wl)
    layers = []
    for _ in range(2):
        lay = DecodeLayer(wl.family, batch, heads, dk, dv, W, st.ranks, B.SS_BF16, **kw)
        lay.load(st.state, st.basis, st.coef, st.A)
        layers.append(lay)
    return wl, st, layers


@pytest.mark.parametrize("family", [synth.MAMBA2, synth.GDN, synth.KDA])
def test_window_replayed_from_a_cuda_graph(cuda_ok, family):
    """A whole window (W-1 decodes and the flush) captured once and replayed
    twice equals the same steps run eagerly, bit for bit."""
    import torch
    wl, st, (eager, graphed) = _pair_of_layers(family)
    W = wl.window
    toks = [eager.token(synth.step_inputs(wl, st, t)) for t in range(W)]
    outs = [torch.empty_like(eager.out) for _ in range(W)]
    for lay in (eager, graphed):
        lay.prime()
    # warm-up window on the layer to be captured (first-call set-up happens here)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for p in range(W):
            graphed.step(toks[p], out=outs[p])
    torch.cuda.current_stream().wait_stream(side)
    for p in range(W):                                       # the eager layer's first window
        eager.step(toks[p])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for p in range(W):
            graphed.step(toks[p], out=outs[p])
    for _ in range(2):
        g.replay()
        ref = []
        for p in range(W):
            eager.step(toks[p])
            ref.append(eager.out.clone())
        torch.cuda.synchronize()
        for p in range(W):
            assert torch.equal(outs[p], ref[p]), f"position {p}: outputs differ"
        assert torch.equal(graphed.state, eager.state)
        assert torch.equal(graphed.sketch, eager.sketch)
        assert torch.equal(graphed.ring_k, eager.ring_k)
    # the graphed plan's phase bookkeeping ran once, at capture; the replays
    # advanced only the device state, window by window
    assert graphed.phase == 0


def test_mixed_step_replayed_from_a_cuda_graph(cuda_ok):
    """The mixed step's fork onto the plan's stream and its join are captured
    with it; replays match eager mixed steps bit for bit."""
    import torch
    wl, st, (eager, graphed) = _pair_of_layers(synth.GDN, W=4, batch=8)
    for lay in (eager, graphed):
        lay.prime()
    tok = eager.token(synth.step_inputs(wl, st, 0))
    fills = [torch.tensor(np.arange(wl.batch) % wl.window, dtype=torch.int32, device="cuda") for _ in range(2)]
    fills_e = [f.clone() for f in fills]
    out_g = torch.empty_like(eager.out)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                            # warm-up: creates the plan's stream
        graphed.step_mixed(tok, fills[0], fills[1], out=out_g)
    torch.cuda.current_stream().wait_stream(side)
    eager.step_mixed(tok, fills_e[0], fills_e[1])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.step_mixed(tok, fills[1], fills[0], out=out_g)
    for k in range(3):
        g.replay()
        eager.step_mixed(tok, fills_e[1], fills_e[0])
        torch.cuda.synchronize()
        assert torch.equal(out_g, eager.out), f"replay {k}: outputs differ"
        assert torch.equal(graphed.state, eager.state) and torch.equal(graphed.ring_k, eager.ring_k)
        assert torch.equal(fills[0], fills_e[0])
        # keep both at the same fills: the graph always reads fills[1] and writes fills[0]
        fills[1].copy_(fills[0])
        fills_e[1].copy_(fills_e[0])


@pytest.mark.parametrize("family", [synth.MAMBA2, synth.GDN])
def test_mixed_steps_with_dense_heads(cuda_ok, family):
    """Mixed window positions with a dense-fallback head beside sketched ones,
    every sequence against its own oracle session."""
    import torch
    W, batch, heads, dk, dv = 4, 6, 3, 128, 64
    wl = synth.Workload(f"mixdense_{family}", family, batch, heads, dk, dv, W, 0, 8, 2700)
    st = synth.static_inputs(wl)
    dense = np.array([0, 1, 0], bool)
    ranks = np.where(dense, dk, st.ranks).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rows = [np.full((dk, dk), np.nan, np.float32) if dense[h] else st.basis[st.offsets[h]:st.offsets[h + 1]]
            for h in range(heads)]
    st.ranks, st.offsets = ranks, offs
    st.basis = np.concatenate(rows).astype(np.float32)
    st.coef = st.basis.copy()
    layer = DecodeLayer(family, batch, heads, dk, dv, W, ranks, dense_heads=dense)
    layer.load(st.state, st.basis, st.coef, st.A)
    sess = [orc.Session(family, st.state[b:b + 1], W, st.A, st.basis, st.coef, st.offsets, dense=dense)
            for b in range(batch)]
    layer.prime()
    for s in sess:
        s.prime()
    fills = (np.arange(batch) % W).astype(np.int32)
    for j in range(W - 1):
        inp = synth.step_inputs(wl, st, 800 + j)
        for b in range(batch):
            if j < fills[b]:
                _put_ring(layer, inp, b, j)
                sess[b].decode(_one(inp, b))
    fin = torch.from_numpy(fills).cuda()
    fout = torch.empty_like(fin)
    fill = fills.copy()
    for t in range(W + 2):
        inp = synth.step_inputs(wl, st, t)
        layer.step_mixed(layer.token(inp), fin, fout)
        torch.cuda.synchronize()
        g = to_np(layer.out)
        for b, s in enumerate(sess):
            o = s.flush(_one(inp, b)) if fill[b] == W - 1 else s.decode(_one(inp, b))[0]
            assert vec_relerr(g[b:b + 1], o) <= TOL, f"seq {b} fill {fill[b]}"
        fill = (fill + 1) % W
        fin, fout = fout, fin
    assert int(layer.status[0].item()) == 0
