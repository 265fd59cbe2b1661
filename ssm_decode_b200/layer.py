"""One layer's decode buffers on the device, driven through the C ABI.

PyTorch only allocates device memory and supplies the stream; every step of
the decode path runs in libsketchssm.so's kernels.  The layout of each buffer
is the one include/sketchssm.h documents.
"""
from __future__ import annotations

import weakref

import numpy as np

from . import binding as B


def _dev(x, dtype, device):
    import torch
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            x = x.view(np.int16)
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.to(device=device, dtype=dtype).contiguous()


class Token(dict):
    """One step's inputs on the device (q, k, v, gate, beta tensors).  The
    C-ABI argument structs built from it are cached per layer, so a step
    costs one library call; update the tensors in place (copy_) to reuse it."""

    def __init__(self, *a, **kw):
        super().__init__(*a, **kw)
        self._io = {}


class DecodeLayer:
    """Plan plus caller-owned device buffers for one linear-attention layer."""

    def __init__(self, family, batch, heads, dk, dv, window, ranks, sketch_dtype=B.SS_F32,
                 device="cuda", coef_mode=B.SS_COEF_FIXED, coef_ridge=0.0, dense_heads=None):
        import torch
        self.plan = B.Plan(family, batch, heads, dk, dv, window, ranks, sketch_dtype, coef_mode, coef_ridge,
                           dense_heads)
        self.family, self.batch, self.heads, self.dk, self.dv, self.window = family, batch, heads, dk, dv, window
        self.device = device
        sz = B.ss_buffer_sizes(self.plan)
        self.R = sz["total_rank"]
        Wg = (window + 3) & ~3
        f32, i16 = torch.float32, torch.int16
        z = lambda *shape, dtype=f32: torch.zeros(shape, dtype=dtype, device=device)
        self.state = z(batch, heads, dk, dv)
        self.ring_k = z(batch, heads, window, dk, dtype=i16)
        self.ring_v = z(batch, heads, window, dv, dtype=i16)
        self.ring_gate = z(batch, heads, window, dk) if family == B.SS_KDA else z(batch, heads, Wg)
        self.ring_beta = None if family == B.SS_MAMBA2 else z(batch, heads, Wg)
        sk_dtype = torch.float32 if sketch_dtype == B.SS_F32 else torch.bfloat16
        self.sketch = torch.zeros((batch, max(self.R, 1), dv), dtype=sk_dtype, device=device)
        self.basis = z(max(self.R, 1), dk)
        self.coef = z(max(self.R, 1), dk)
        # per-(sequence, head) coefficient maps of SS_COEF_STATE / SS_COEF_LRD, sketch dtype
        self.coef_state = (torch.zeros((batch, max(self.R, 1), dk), dtype=sk_dtype, device=device)
                           if coef_mode in (B.SS_COEF_STATE, B.SS_COEF_LRD) else None)
        self.A = z(heads)
        self.out = z(batch, heads, dv)
        self.status = torch.zeros(4, dtype=torch.int32, device=device)   # device status word (+ padding)
        self.sketch_dtype = sketch_dtype
        # The buffers stay in place for the layer's life (load() copies into
        # them), so their argument structs are built once.
        self._bufs = {w: self._make_bufs(w) for w in (True, False)}

    # -- data -------------------------------------------------------------------
    def load(self, state=None, basis=None, coef=None, A=None):
        if state is not None:
            self.state.copy_(_dev(state, self.state.dtype, self.device))
        if basis is not None and self.R:
            self.basis.copy_(_dev(basis, self.basis.dtype, self.device))
        if coef is not None and self.R:
            self.coef.copy_(_dev(coef, self.coef.dtype, self.device))
        if A is not None:
            self.A.copy_(_dev(A, self.A.dtype, self.device))

    def token(self, inp):
        """Move one step's raw inputs (numpy or torch) to the device."""
        import torch
        t = Token((k, _dev(inp[k], torch.int16, self.device)) for k in ("q", "k", "v"))
        t["gate"] = _dev(inp["gate"], torch.float32, self.device)
        t["beta"] = _dev(inp["beta"], torch.float32, self.device)
        return t

    def bufs(self, with_sketch=True):
        return self._bufs[bool(with_sketch)]

    def _make_bufs(self, with_sketch):
        return B.make_buffers(self.state, self.ring_k, self.ring_v, self.ring_gate, self.ring_beta,
                              self.sketch if with_sketch else None, self.basis, self.coef, self.A,
                              self.status, self.coef_state)

    def io(self, tok, out=None):
        cache = getattr(tok, "_io", None) if out is None else None
        if cache is not None:
            hit = cache.get(id(self))
            if hit is not None and hit[0]() is self:      # guard against a reused id()
                return hit[1]
        beta = tok["beta"] if self.family != B.SS_MAMBA2 else None
        io = B.make_step_io(tok["q"], tok["k"], tok["v"], tok["gate"], beta,
                            self.out if out is None else out)
        if cache is not None:
            cache[id(self)] = (weakref.ref(self), io)
        return io

    @property
    def phase(self):
        return B.ss_get_phase(self.plan)[0]

    # -- calls --------------------------------------------------------------------
    def prime(self, stream=None):
        B.ss_prime(self.plan, self.bufs(), stream)

    def decode(self, tok, out=None, stream=None):
        B.ss_decode_step(self.plan, self.bufs(), self.io(tok, out), stream)

    def flush(self, tok=None, with_sketch=True, out=None, stream=None):
        io = None if tok is None else self.io(tok, out)
        B.ss_flush(self.plan, self.bufs(with_sketch), io, stream)

    def step(self, tok, out=None, stream=None):
        """One SketchSSM step: non-flush until the window's last token, then flush."""
        if self.phase == self.window - 1:
            self.flush(tok, out=out, stream=stream)
        else:
            self.decode(tok, out=out, stream=stream)

    def exact_step(self, tok, out=None, stream=None):
        B.ss_exact_step(self.plan, self.bufs(False), self.io(tok, out), stream)

    def step_mixed(self, tok, fill_in, fill_out, out=None, stream=None):
        """One step with a window position per sequence (int32 device tensors
        of `batch` entries): sequences at W-1 flush, the rest decode;
        fill_out receives (fill_in + 1) mod W."""
        B.ss_step_mixed(self.plan, self.bufs(), self.io(tok, out), fill_in, fill_out, stream)

    def replay_step(self, tok, out=None, stream=None):
        if self.phase == self.window - 1:
            self.flush(tok, with_sketch=False, out=out, stream=stream)
        else:
            B.ss_replay_step(self.plan, self.bufs(False), self.io(tok, out), stream)
