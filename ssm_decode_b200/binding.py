"""ctypes binding of libsketchssm.so (include/sketchssm.h), same names as the C ABI.

Argument marshalling only: torch tensors are turned into device pointers and
the current CUDA stream into an ss_stream; every step of the decode path runs
in the library's kernels.  If the library is missing, importing the functions
raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsketchssm.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "sketchssm.h")

SS_OK, SS_ERR_INVALID_ARG, SS_ERR_ALIGNMENT, SS_ERR_UNSUPPORTED, SS_ERR_SCHEDULE, SS_ERR_CUDA = range(6)
SS_DEVICE_TIMEOUT = 1
SS_DEVICE_BAD_FILL = 2
SS_DEVICE_SINGULAR_MAP = 4
SS_COEF_FIXED, SS_COEF_STATE, SS_COEF_LRD = 0, 1, 2
SS_MAMBA2, SS_GDN, SS_KDA = 0, 1, 2
SS_F32, SS_BF16 = 0, 1
(SS_OP_DECODE, SS_OP_FLUSH, SS_OP_FLUSH_NO_TOKEN, SS_OP_PRIME, SS_OP_EXACT, SS_OP_REPLAY,
 SS_OP_REPLAY_FLUSH) = range(7)


class ss_config(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int32), ("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("window", ctypes.c_int32),
                ("ranks", ctypes.POINTER(ctypes.c_int32)), ("sketch_dtype", ctypes.c_int32),
                ("coef_mode", ctypes.c_int32), ("coef_ridge", ctypes.c_float),
                ("dense_heads", ctypes.POINTER(ctypes.c_uint8))]


class ss_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("state", "ring_k", "ring_v", "ring_gate", "ring_beta", "sketch", "basis", "coef", "A",
                 "q", "k", "v", "gate", "beta", "out", "coef_state")] + \
               [("total_rank", ctypes.c_int32), ("gate_stride", ctypes.c_int32)]


class ss_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("state", "ring_k", "ring_v", "ring_gate", "ring_beta", "sketch", "basis", "coef", "A",
                 "status", "coef_state")]


class ss_step_io(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "gate", "beta", "out")]


class ss_traffic(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in
                ("paper_read_bytes", "paper_write_bytes", "read_bytes", "write_bytes")]


class SSError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_name(status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m ssm_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.c_int
        sig = {
            "ss_create": ([ctypes.POINTER(ss_config), ctypes.POINTER(P)], S),
            "ss_destroy": ([P], S),
            "ss_buffer_sizes": ([P, ctypes.POINTER(ss_sizes)], S),
            "ss_get_phase": ([P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)], S),
            "ss_set_phase": ([P, ctypes.c_int32, ctypes.c_int32], S),
            "ss_prime": ([P, ctypes.POINTER(ss_buffers), P], S),
            "ss_decode_step": ([P, ctypes.POINTER(ss_buffers), ctypes.POINTER(ss_step_io), P], S),
            "ss_flush": ([P, ctypes.POINTER(ss_buffers), ctypes.POINTER(ss_step_io), P], S),
            "ss_exact_step": ([P, ctypes.POINTER(ss_buffers), ctypes.POINTER(ss_step_io), P], S),
            "ss_replay_step": ([P, ctypes.POINTER(ss_buffers), ctypes.POINTER(ss_step_io), P], S),
            "ss_step_mixed": ([P, ctypes.POINTER(ss_buffers), ctypes.POINTER(ss_step_io), P, P, P], S),
            "ss_traffic_bytes": ([P, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ss_traffic)], S),
            "ss_launch_count": ([], ctypes.c_uint64),
            "ss_debug_stall_next_copy": ([P, ctypes.c_int32], S),
            "ss_debug_fail_launch": ([P, ctypes.c_int32], S),
            "ss_status_string": ([S], ctypes.c_char_p),
            "ss_last_error_string": ([], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes, fn.restype = args, res
        _lib = L
    return _lib


def header_functions():
    """Names of the functions include/sketchssm.h declares."""
    with open(HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(ss_[a-z_]+)\s*\(", text)) - {"ss_stream"})


def status_name(s):
    try:
        return lib().ss_status_string(s).decode()
    except ImportError:
        return str(s)


def _check(status):
    if status != SS_OK:
        raise SSError(status, lib().ss_last_error_string().decode())


# ---------------------------------------------------------------------------
# tensor -> pointer marshalling
# ---------------------------------------------------------------------------
def _ptr(t, what, dtypes=None):
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a torch.Tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{what}: dtype {t.dtype} not in {dtypes}")
    if not t.is_cuda:
        raise ValueError(f"{what}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")
    return t.data_ptr()


def _dt():
    import torch
    return {"f32": (torch.float32,), "bf16": (torch.bfloat16, torch.int16, torch.uint16),
            "any": None}


def make_buffers(state=None, ring_k=None, ring_v=None, ring_gate=None, ring_beta=None, sketch=None,
                 basis=None, coef=None, A=None, status=None, coef_state=None):
    import torch
    d = _dt()
    return ss_buffers(_ptr(state, "state", d["f32"]), _ptr(ring_k, "ring_k", d["bf16"]),
                      _ptr(ring_v, "ring_v", d["bf16"]), _ptr(ring_gate, "ring_gate", d["f32"]),
                      _ptr(ring_beta, "ring_beta", d["f32"]),
                      _ptr(sketch, "sketch", d["f32"] + d["bf16"]), _ptr(basis, "basis", d["f32"]),
                      _ptr(coef, "coef", d["f32"]), _ptr(A, "A", d["f32"]),
                      _ptr(status, "status", (torch.int32,)),
                      _ptr(coef_state, "coef_state", d["f32"] + d["bf16"]))


def make_step_io(q, k, v, gate, beta, out):
    d = _dt()
    return ss_step_io(_ptr(q, "q", d["bf16"]), _ptr(k, "k", d["bf16"]), _ptr(v, "v", d["bf16"]),
                      _ptr(gate, "gate", d["f32"]), _ptr(beta, "beta", d["f32"]),
                      _ptr(out, "out", d["f32"]))


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ---------------------------------------------------------------------------
# the ABI, one wrapper per entry point
# ---------------------------------------------------------------------------
class Plan:
    """Owns an ss_plan*; destroyed with the object."""

    def __init__(self, family, batch, heads, dk, dv, window, ranks, sketch_dtype=SS_F32,
                 coef_mode=SS_COEF_FIXED, coef_ridge=0.0, dense_heads=None):
        self.ranks = (ctypes.c_int32 * heads)(*[int(r) for r in ranks])
        self.dense_heads = None if dense_heads is None else (ctypes.c_uint8 * heads)(*[int(bool(d)) for d in dense_heads])
        cfg = ss_config(family, batch, heads, dk, dv, window,
                        ctypes.cast(self.ranks, ctypes.POINTER(ctypes.c_int32)), sketch_dtype,
                        coef_mode, coef_ridge,
                        None if self.dense_heads is None
                        else ctypes.cast(self.dense_heads, ctypes.POINTER(ctypes.c_uint8)))
        h = ctypes.c_void_p()
        _check(lib().ss_create(ctypes.byref(cfg), ctypes.byref(h)))
        self.handle = h
        self.family, self.batch, self.heads, self.dk, self.dv, self.window = family, batch, heads, dk, dv, window
        self.sketch_dtype = sketch_dtype
        self.coef_mode, self.coef_ridge = coef_mode, coef_ridge

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _lib is not None:
            _lib.ss_destroy(h)
            self.handle = None


def ss_create(family, batch, heads, dk, dv, window, ranks, sketch_dtype=SS_F32, coef_mode=SS_COEF_FIXED,
              coef_ridge=0.0):
    return Plan(family, batch, heads, dk, dv, window, ranks, sketch_dtype, coef_mode, coef_ridge)


def ss_buffer_sizes(plan):
    s = ss_sizes()
    _check(lib().ss_buffer_sizes(plan.handle, ctypes.byref(s)))
    return {n: getattr(s, n) for n, _ in ss_sizes._fields_}


def ss_get_phase(plan):
    ph, sv = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().ss_get_phase(plan.handle, ctypes.byref(ph), ctypes.byref(sv)))
    return ph.value, bool(sv.value)


def ss_set_phase(plan, phase, sketch_valid):
    _check(lib().ss_set_phase(plan.handle, phase, int(bool(sketch_valid))))


def ss_prime(plan, bufs, stream=None):
    _check(lib().ss_prime(plan.handle, ctypes.byref(bufs), _stream(stream)))


def ss_decode_step(plan, bufs, io, stream=None):
    _check(lib().ss_decode_step(plan.handle, ctypes.byref(bufs), ctypes.byref(io), _stream(stream)))


def ss_flush(plan, bufs, io=None, stream=None):
    iop = ctypes.byref(io) if io is not None else None
    _check(lib().ss_flush(plan.handle, ctypes.byref(bufs), iop, _stream(stream)))


def ss_exact_step(plan, bufs, io, stream=None):
    _check(lib().ss_exact_step(plan.handle, ctypes.byref(bufs), ctypes.byref(io), _stream(stream)))


def ss_replay_step(plan, bufs, io, stream=None):
    _check(lib().ss_replay_step(plan.handle, ctypes.byref(bufs), ctypes.byref(io), _stream(stream)))


def ss_step_mixed(plan, bufs, io, fill_in, fill_out, stream=None):
    """fill_in / fill_out: device int32 tensors of `batch` entries (or raw pointers)."""
    fi = fill_in if isinstance(fill_in, int) else fill_in.data_ptr()
    fo = fill_out if isinstance(fill_out, int) else fill_out.data_ptr()
    _check(lib().ss_step_mixed(plan.handle, ctypes.byref(bufs), ctypes.byref(io), fi, fo, _stream(stream)))


def ss_traffic_bytes(plan, op, tau=0):
    t = ss_traffic()
    _check(lib().ss_traffic_bytes(plan.handle, op, tau, ctypes.byref(t)))
    return {n: getattr(t, n) for n, _ in ss_traffic._fields_}


def ss_launch_count():
    return int(lib().ss_launch_count())


def ss_debug_stall_next_copy(plan, stall=True):
    _check(lib().ss_debug_stall_next_copy(plan.handle, int(bool(stall))))


def ss_debug_fail_launch(plan, n):
    """Testing hook: the n-th launch of this plan's next calls is refused on the host."""
    _check(lib().ss_debug_fail_launch(plan.handle, int(n)))


def ss_status_string(s):
    return lib().ss_status_string(s).decode()


def ss_last_error_string():
    return lib().ss_last_error_string().decode()
