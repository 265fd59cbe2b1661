"""Out-of-bounds write detection without a sanitizer: canary-padded buffers.

Every device buffer the library reads or writes (state, ring, sketch, maps,
basis, outputs, fills, status, the step's inputs) is a view into a larger
tensor whose head and tail are filled with a fixed bit pattern.  After tiny
cases exercising every call (prime, decode, flush with and without a token,
mixed steps, replay, the Standard step, the state-dependent map, dense heads)
the patterns must be intact.
"""
import numpy as np
import pytest

from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from ssm_decode_b200.layer import DecodeLayer, Token

pytestmark = pytest.mark.gpu

PAD = 4096          # bytes of canary before and after each buffer (a multiple of 16)
PATTERN = 0x5A3CC3A5


class Guarded:
    """Padded allocations; view(t) returns a same-shape tensor inside a canary."""

    def __init__(self):
        self.blocks = []

    def view(self, t):
        import torch
        nbytes = t.numel() * t.element_size()
        words = (2 * PAD + ((nbytes + 15) // 16) * 16) // 4
        raw = torch.full((words,), PATTERN - (1 << 32) if PATTERN >= (1 << 31) else PATTERN,
                         dtype=torch.int32, device=t.device)
        body = raw[PAD // 4:PAD // 4 + (nbytes + 3) // 4]
        v = body.view(torch.uint8)[:nbytes].view(t.dtype).view(t.shape)
        v.copy_(t)
        self.blocks.append((raw, nbytes))
        return v

    def check(self):
        import torch
        if torch.cuda.is_available():
            torch.cuda.synchronize()
        for raw, nbytes in self.blocks:
            w = raw.cpu().numpy().view(np.uint32)
            head = w[:PAD // 4]
            tail_start = PAD // 4 + (nbytes + 3) // 4
            assert (head == PATTERN).all(), "a write landed before a buffer"
            # the bytes between the end of the data and the next word keep the pattern too
            tail = w[((PAD + nbytes + 15) // 16) * 4:]
            assert (tail == PATTERN).all(), "a write landed after a buffer"
            assert tail_start <= len(w)


def guard_layer(lay, g):
    for name in ("state", "ring_k", "ring_v", "ring_gate", "ring_beta", "sketch", "basis", "coef", "A", "out",
                 "status", "coef_state"):
        t = getattr(lay, name, None)
        if t is not None:
            setattr(lay, name, g.view(t))
    lay._bufs = {w: lay._make_bufs(w) for w in (True, False)}


def guard_token(tok, g):
    return Token({k: g.view(v) for k, v in tok.items()})


@pytest.mark.parametrize("family", [synth.MAMBA2, synth.GDN, synth.KDA])
@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128)])
def test_no_write_outside_any_buffer(cuda_ok, family, dk, dv):
    import torch
    W, batch, heads = 5, 3, 4
    wl = synth.Workload("canary", family, batch, heads, dk, dv, W, 0, 8, 3000 + dk)
    st = synth.static_inputs(wl)
    ranks = np.array([0, 1, 16, 5], np.int32)
    offs = np.concatenate([[0], np.cumsum(ranks)]).astype(np.int32)
    rng = np.random.default_rng(30)
    basis = np.concatenate([np.linalg.qr(rng.standard_normal((dk, dk)))[0][:, :r].T for r in ranks]).astype(np.float32)
    g = Guarded()
    layers = []
    for kw in ({}, {"coef_mode": B.SS_COEF_STATE, "coef_ridge": 0.1},
               {"dense_heads": [0, 0, 0, 1]}):
        rk = ranks if "dense_heads" not in kw else np.where(np.array(kw["dense_heads"], bool), dk, ranks)
        bs = basis if "dense_heads" not in kw else np.concatenate(
            [basis[offs[h]:offs[h + 1]] if not kw["dense_heads"][h] else np.eye(dk, dtype=np.float32)
             for h in range(heads)])
        lay = DecodeLayer(family, batch, heads, dk, dv, W, rk, B.SS_BF16, **kw)
        lay.load(st.state, bs, bs, st.A)
        guard_layer(lay, g)
        layers.append(lay)
    toks = [guard_token(layers[0].token(synth.step_inputs(wl, st, t)), g) for t in range(2 * W + 2)]
    fills = [g.view(torch.tensor(np.arange(batch) % W, dtype=torch.int32, device="cuda")),
             g.view(torch.zeros(batch, dtype=torch.int32, device="cuda"))]
    for lay in layers:
        lay.prime()
        for t in range(W + 2):                       # a window, its flush, then two decodes
            lay.step(toks[t])
        lay.flush(None)                              # end of sequence: the buffered updates only
        lay.prime()
        for t in range(3):                           # mixed positions, both fill buffers
            lay.step_mixed(toks[t], fills[t % 2], fills[1 - t % 2])
        for t in range(W):                           # ReplaySSM window (its flush keeps no sketch)
            lay.replay_step(toks[t])
        lay.exact_step(toks[0])                      # Standard step
        lay.prime()
    g.check()
    assert all(int(l.status[0].item()) == 0 for l in layers)
