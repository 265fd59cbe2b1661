"""Shared helpers of the GPU parity tests: run the CUDA library and the fp64
oracle side by side on the same seeded inputs and compare.

Tolerances (fp32 state and arithmetic, bf16 q/k/v):
  * outputs, states, fp32 sketches: per vector / per head,
    max|gpu - oracle| / max|oracle| <= 1e-4;
  * bf16 sketch: every element within a(u) = one bf16 ulp of the oracle's
    rounded value + 1e-4 of the head's largest sketch entry (fp32 rounding
    and ties straddled by fp32 and fp64), and each sketched output element
    within 1e-4 max|o| + sum_i |c_i| a(u_i[v]) of the oracle's;
  * ring buffer: bit-exact.
"""
import numpy as np

from oracle import sketchssm_oracle as orc
from ssm_decode_b200 import binding as B
from ssm_decode_b200 import synth
from ssm_decode_b200.layer import DecodeLayer

TOL = 1e-4


def vec_relerr(g, o):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    num = np.abs(g - o).max(axis=-1)
    den = np.maximum(np.abs(o).max(axis=-1), 1e-30)
    return float((num / den).max())


def head_relerr(g, o):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    num = np.abs(g - o).max(axis=(-2, -1))
    den = np.maximum(np.abs(o).max(axis=(-2, -1)), 1e-30)
    return float((num / den).max())


def bf16_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.where(x > 0, x, 1.0))
    return np.ldexp(1.0, np.maximum(e - 8, -133))


def to_np(t):
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    if t.dtype == torch.int16:
        return t.numpy().view(np.uint16)
    return t.numpy()


class Pair:
    """A DecodeLayer on the GPU and an oracle Session fed the same bytes.

    ``sel`` restricts the oracle to a subset of sequences (full-size runs
    compare sampled sequences); the GPU always runs the whole batch.
    """

    def __init__(self, wl, st=None, sketch_dtype=B.SS_F32, sel=None, state_map=False, rho=0.0, dense=None,
                 map_kind="exact"):
        import torch
        self.wl = wl
        self.st = st if st is not None else synth.static_inputs(wl)
        self.sel = np.arange(wl.batch) if sel is None else np.asarray(sel)
        self.state_map, self.map_kind = state_map, map_kind
        mode = (B.SS_COEF_LRD if map_kind == "lrd" else B.SS_COEF_STATE) if state_map else B.SS_COEF_FIXED
        self.layer = DecodeLayer(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, wl.window,
                                 self.st.ranks, sketch_dtype,
                                 coef_mode=mode,
                                 coef_ridge=rho, dense_heads=dense)
        self.layer.load(self.st.state, self.st.basis, self.st.coef, self.st.A)
        self.sess = orc.Session(wl.family, self.st.state[self.sel], wl.window, self.st.A,
                                self.st.basis, self.st.coef, self.st.offsets,
                                sketch_bf16=sketch_dtype == B.SS_BF16, state_map=state_map, rho=rho,
                                dense=dense, map_kind=map_kind)
        self.bf16 = sketch_dtype == B.SS_BF16
        self.ring_k = np.zeros((wl.batch, wl.heads, wl.window, wl.dk), np.uint16)
        self.ring_v = np.zeros((wl.batch, wl.heads, wl.window, wl.dv), np.uint16)
        self.worst = {"out": 0.0, "sketched": 0.0, "state": 0.0, "sketch": 0.0, "map": 0.0}
        torch.cuda.synchronize()

    # -- checks ------------------------------------------------------------------
    def out(self):
        import torch
        torch.cuda.synchronize()
        return to_np(self.layer.out)[self.sel]

    def check_state(self):
        err = head_relerr(to_np(self.layer.state)[self.sel], self.sess.S)
        self.worst["state"] = max(self.worst["state"], err)
        assert err <= TOL, f"state relerr {err:.3e}"

    def check_sketch(self):
        g = to_np(self.layer.sketch)[self.sel]
        ref = self.sess.packed_sketch()
        if self.bf16:
            ok = np.abs(g - ref) <= self._sketch_allowance(ref) * (1 + 1e-9)
            assert ok.all(), f"{(~ok).sum()} sketch entries beyond one bf16 ulp + fp32 allowance"
            self.worst["sketch"] = max(self.worst["sketch"], float(np.mean(g != ref)))
        else:
            offs = self.st.offsets
            for h in range(self.wl.heads):
                if offs[h + 1] == offs[h]:
                    continue
                err = head_relerr(g[:, offs[h]:offs[h + 1]], ref[:, offs[h]:offs[h + 1]])
                self.worst["sketch"] = max(self.worst["sketch"], err)
                assert err <= TOL, f"sketch head {h} relerr {err:.3e}"

    def gpu_sketch_heads(self):
        """The GPU's stored sketch per head, widened: list of [b, V, r_h]."""
        u = to_np(self.layer.sketch)[self.sel]
        offs = self.st.offsets
        return [np.transpose(u[:, offs[h]:offs[h + 1]], (0, 2, 1)) for h in range(self.wl.heads)]

    def check_map(self):
        """State-dependent maps: per head, max|gpu - oracle| / max|oracle| within
        1e-4 (fp32).  With a bf16 sketch the map is a function of the stored U,
        whose entries may sit one bf16 ulp from the oracle's rounding (fp32 vs
        fp64 straddling a tie), and the solve amplifies that; so the reference
        map is the oracle's map of the GPU's own stored U (reading P7), rounded
        to bf16, and each entry must lie within one bf16 ulp of it plus 1e-4
        of the head's largest entry."""
        if not self.state_map:
            return
        g = to_np(self.layer.coef_state)[self.sel]
        if self.bf16 and self.map_kind == "lrd":
            ref = self.sess.packed_map()     # a function of the state alone: the oracle's, rounded
        elif self.bf16:
            Ug = self.gpu_sketch_heads()
            ref = np.concatenate([np.zeros((len(self.sel), self.wl.dk, self.wl.dk)) if self.sess.dense[h] else
                                  orc.round_bf16(orc.coefficient_map(Ug[h], self.sess.S[:, h], self.sess.rho))
                                  for h in range(self.wl.heads)], axis=1)
        else:
            ref = self.sess.packed_map()
        offs = self.st.offsets
        for h in range(self.wl.heads):
            if offs[h + 1] == offs[h] or self.sess.dense[h]:     # a dense head has no map
                continue
            gh, rh = g[:, offs[h]:offs[h + 1]], ref[:, offs[h]:offs[h + 1]]
            if self.bf16:
                allow = bf16_ulp(rh) + TOL * np.abs(rh).max(axis=(1, 2), keepdims=True)
                ok = np.abs(gh - rh) <= allow * (1 + 1e-9)
                assert ok.all(), f"map head {h}: {(~ok).sum()} entries beyond one bf16 ulp + allowance"
            else:
                err = head_relerr(gh, rh)
                self.worst["map"] = max(self.worst["map"], err)
                assert err <= TOL, f"map head {h} relerr {err:.3e}"

    def check_ring(self):
        ph = self.layer.phase
        gk = to_np(self.layer.ring_k)
        gv = to_np(self.layer.ring_v)
        assert np.array_equal(gk[:, :, :ph], self.ring_k[:, :, :ph]), "ring keys differ"
        assert np.array_equal(gv[:, :, :ph], self.ring_v[:, :, :ph]), "ring values differ"

    def _sketch_allowance(self, ref):
        """One bf16 ulp of the rounded value, plus the fp32 tolerance relative to the
        head's largest sketch entry (entries near zero come from cancelling sums whose
        fp32 rounding error can exceed a bf16 ulp of the tiny result)."""
        allow = bf16_ulp(ref)
        offs = self.st.offsets
        for h in range(self.wl.heads):
            blk = ref[:, offs[h]:offs[h + 1]]
            if blk.size:
                allow[:, offs[h]:offs[h + 1]] += TOL * np.abs(blk).max(axis=(1, 2), keepdims=True)
        return allow

    # -- steps -------------------------------------------------------------------------
    def prime(self):
        self.layer.prime()
        self.sess.prime()
        self.check_sketch()
        self.check_map()

    def _sub(self, inp):
        return {k: v[self.sel] for k, v in inp.items()}

    def _record(self, inp, slot):
        self.ring_k[:, :, slot] = inp["k"]
        self.ring_v[:, :, slot] = inp["v"]

    def step(self, inp, ring=True):
        """One SketchSSM step on both sides; compare."""
        tok = self.layer.token(inp)
        ph = self.layer.phase
        self.layer.step(tok)
        g = self.out()
        if ph == self.wl.window - 1:
            o = self.sess.flush(self._sub(inp))
            err = vec_relerr(g, o)
            self.worst["out"] = max(self.worst["out"], err)
            assert err <= TOL, f"flush output relerr {err:.3e}"
            self.check_state()
            self.check_sketch()
            self.check_map()
        else:
            o_hat, _ = self.sess.decode(self._sub(inp))
            if self.bf16 and self.state_map:
                # the GPU's stored bf16 U and map applied to the oracle's q~ and buffered term
                Cg = to_np(self.layer.coef_state)[self.sel]
                Ug = self.gpu_sketch_heads()
                offs = self.st.offsets
                ref = np.empty_like(o_hat)
                for h in range(self.wl.heads):
                    if self.sess.dense[h]:                               # the identity map
                        c = self.sess.last_q_tilde[:, h]
                    else:
                        c = np.einsum("brk,bk->br", Cg[:, offs[h]:offs[h + 1]], self.sess.last_q_tilde[:, h])
                    ref[:, h] = np.einsum("bvr,br->bv", Ug[h], c) + self.sess.last_o_buf[:, h]
                err = vec_relerr(g, ref)
                self.worst["sketched"] = max(self.worst["sketched"], err)
                assert err <= TOL, f"sketched output (stored bf16 U and map) relerr {err:.3e} at phase {ph}"
            elif self.bf16:
                ref_u = self.sess.packed_sketch()
                allow_u = self._sketch_allowance(ref_u)
                bound = np.broadcast_to(TOL * np.abs(o_hat).max(-1, keepdims=True), o_hat.shape).copy()
                offs = self.st.offsets
                for h in range(self.wl.heads):
                    c = self.sess.last_coefficients[h]                       # [b, r]
                    u = allow_u[:, offs[h]:offs[h + 1]]                      # [b, r, V]
                    bound[:, h] += np.einsum("br,brv->bv", np.abs(c), u)
                excess = np.abs(g - o_hat) - bound * (1 + 1e-6)
                assert (excess <= 0).all(), f"sketched output beyond bound by {excess.max():.3e}"
                self.worst["sketched"] = max(self.worst["sketched"], vec_relerr(g, o_hat))
            else:
                err = vec_relerr(g, o_hat)
                self.worst["sketched"] = max(self.worst["sketched"], err)
                assert err <= TOL, f"sketched output relerr {err:.3e} at phase {ph}"
            if ring:
                self._record(inp, ph)
                self.check_ring()

    def exact_step(self, inp):
        tok = self.layer.token(inp)
        self.layer.exact_step(tok)
        g = self.out()
        o = self.sess.exact_step(self._sub(inp))
        err = vec_relerr(g, o)
        self.worst["out"] = max(self.worst["out"], err)
        assert err <= TOL, f"exact-step output relerr {err:.3e}"
        self.check_state()

    def replay_step(self, inp):
        tok = self.layer.token(inp)
        ph = self.layer.phase
        self.layer.replay_step(tok)
        g = self.out()
        if ph == self.wl.window - 1:
            o = self.sess.flush(self._sub(inp), with_sketch=False)
            self.check_state()
        else:
            o = self.sess.replay_step(self._sub(inp))
            self._record(inp, ph)
            self.check_ring()
        err = vec_relerr(g, o)
        self.worst["out"] = max(self.worst["out"], err)
        assert err <= TOL, f"replay output relerr {err:.3e} at phase {ph}"
