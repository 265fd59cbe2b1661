"""Host-side checks of libsketchssm.so that need no GPU.

The library must load, export every function include/sketchssm.h declares,
reject bad shapes, pointers and out-of-order calls before launching anything,
and reproduce the pages' printed traffic-reduction figures from its traffic
model.  Calls here never pass validation with fake pointers: every one is
built to fail a check first (and the fake-pointer tests skip on a GPU host).
"""
import ctypes
import json
import os

import pytest

from ssm_decode_b200 import binding as B
from ssm_decode_b200 import build

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def L():
    build.build()
    return B.lib()


def _no_gpu():
    import torch
    return not torch.cuda.is_available()


def test_exports_every_header_symbol(L):
    names = B.header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/sketchssm.h but not exported"


def test_create_rejects_bad_shapes(L):
    def code(**kw):
        cfg = dict(family=0, batch=2, heads=3, dk=64, dv=64, window=16, ranks=[4, 4, 4], sketch_dtype=0)
        cfg.update(kw)
        try:
            B.Plan(cfg["family"], cfg["batch"], cfg["heads"], cfg["dk"], cfg["dv"], cfg["window"],
                   cfg["ranks"], cfg["sketch_dtype"])
            return B.SS_OK
        except B.SSError as e:
            return e.status
    assert code() == B.SS_OK
    assert code(family=3) == B.SS_ERR_INVALID_ARG
    assert code(batch=0) == B.SS_ERR_INVALID_ARG
    assert code(dk=96) == B.SS_ERR_UNSUPPORTED
    assert code(dv=32) == B.SS_ERR_UNSUPPORTED
    assert code(window=0) == B.SS_ERR_UNSUPPORTED
    assert code(window=33) == B.SS_ERR_UNSUPPORTED
    assert code(ranks=[4, 65, 4]) == B.SS_ERR_INVALID_ARG
    assert code(ranks=[4, -1, 4]) == B.SS_ERR_INVALID_ARG
    assert code(sketch_dtype=7) == B.SS_ERR_INVALID_ARG
    assert code(heads=513, ranks=[1] * 513) == B.SS_ERR_UNSUPPORTED
    assert code(window=1) == B.SS_OK and code(ranks=[0, 64, 1]) == B.SS_OK


def test_supported_rank_and_window_range(L):
    """The shared-memory limits stated for ss_create: every rank up to 64 at
    W <= 16 and up to 32 at W <= 32 is accepted, for every family, shape and
    sketch type; KDA with rank 128, dk = dv = 128 and W = 32 is not."""
    def ok(fam, dk, dv, W, r, sk):
        try:
            B.Plan(fam, 2, 2, dk, dv, W, [r, 1], sk)
            return True
        except B.SSError as e:
            assert e.status == B.SS_ERR_UNSUPPORTED
            return False
    for fam in (B.SS_MAMBA2, B.SS_GDN, B.SS_KDA):
        for dk, dv in ((64, 64), (64, 128), (128, 64), (128, 128)):
            for sk in (B.SS_F32, B.SS_BF16):
                assert ok(fam, dk, dv, 16, min(64, dk), sk)
                assert ok(fam, dk, dv, 32, 32, sk)
    assert not ok(B.SS_KDA, 128, 128, 32, 128, B.SS_F32)


def test_buffer_sizes(L):
    p = B.Plan(B.SS_KDA, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16)
    s = B.ss_buffer_sizes(p)
    assert s["state"] == 3 * 2 * 128 * 64 * 4
    assert s["ring_k"] == 3 * 2 * 6 * 128 * 2 and s["ring_v"] == 3 * 2 * 6 * 64 * 2
    assert s["ring_gate"] == 3 * 2 * 6 * 128 * 4          # KDA: per-channel decays
    assert s["ring_beta"] == 3 * 2 * 8 * 4                  # W rounded up to 8
    assert s["sketch"] == 3 * 12 * 64 * 2 and s["basis"] == 12 * 128 * 4
    assert s["total_rank"] == 12 and s["gate_stride"] == 6 * 128
    m = B.ss_buffer_sizes(B.Plan(B.SS_MAMBA2, 1, 4, 64, 64, 5, [1, 2, 3, 4]))
    assert m["ring_gate"] == 4 * 8 * 4 and m["ring_beta"] == 0 and m["A"] == 16


def _fake_bufs(bad=None, null=None):
    vals = {n: 0x10000 * (i + 1) for i, (n, _) in enumerate(B.ss_buffers._fields_)}
    if bad:
        vals[bad] += 4
    if null:
        vals[null] = None
    return B.ss_buffers(*[vals[n] for n, _ in B.ss_buffers._fields_])


def _fake_io(bad=None, null=None):
    vals = {n: 0x900000 + 0x10000 * i for i, (n, _) in enumerate(B.ss_step_io._fields_)}
    if bad:
        vals[bad] += 8
    if null:
        vals[null] = None
    return B.ss_step_io(*[vals[n] for n, _ in B.ss_step_io._fields_])


@pytest.mark.skipif(not _no_gpu(), reason="fake-pointer validation tests run on CPU hosts only")
def test_schedule_and_argument_errors(L):
    p = B.Plan(B.SS_GDN, 2, 2, 64, 64, 4, [2, 3])
    st = ctypes.c_void_p(0)
    bufs, io = _fake_bufs(bad="state"), _fake_io()

    def rc(fn, *args):
        return fn(p.handle, *args)

    # schedule errors come first, before any pointer is looked at
    assert rc(L.ss_decode_step, ctypes.byref(bufs), ctypes.byref(io), st) == B.SS_ERR_SCHEDULE  # no sketch yet
    assert rc(L.ss_flush, ctypes.byref(bufs), ctypes.byref(io), st) == B.SS_ERR_SCHEDULE        # phase 0 != W-1
    B.ss_set_phase(p, 3, True)
    assert rc(L.ss_decode_step, ctypes.byref(bufs), ctypes.byref(io), st) == B.SS_ERR_SCHEDULE  # must flush now
    assert rc(L.ss_replay_step, ctypes.byref(bufs), ctypes.byref(io), st) == B.SS_ERR_SCHEDULE
    assert rc(L.ss_prime, ctypes.byref(bufs), st) == B.SS_ERR_SCHEDULE
    assert rc(L.ss_exact_step, ctypes.byref(bufs), ctypes.byref(io), st) == B.SS_ERR_SCHEDULE
    assert "phase" in B.ss_last_error_string()
    assert B.ss_get_phase(p) == (3, True)
    # pointer checks at a legal phase: NULL -> INVALID_ARG, misaligned -> ALIGNMENT
    B.ss_set_phase(p, 1, True)
    for name in ("state", "ring_k", "ring_v", "ring_gate", "ring_beta", "sketch", "coef"):
        b = _fake_bufs(bad=name)
        assert rc(L.ss_decode_step, ctypes.byref(b), ctypes.byref(io), st) == B.SS_ERR_ALIGNMENT, name
        b = _fake_bufs(null=name)
        assert rc(L.ss_decode_step, ctypes.byref(b), ctypes.byref(io), st) == B.SS_ERR_INVALID_ARG, name
    for name in ("q", "k", "v", "gate", "beta", "out"):
        i2 = _fake_io(bad=name)
        assert rc(L.ss_decode_step, ctypes.byref(_fake_bufs()), ctypes.byref(i2), st) == B.SS_ERR_ALIGNMENT
        i2 = _fake_io(null=name)
        assert rc(L.ss_replay_step, ctypes.byref(_fake_bufs()), ctypes.byref(i2), st) == B.SS_ERR_INVALID_ARG
    assert rc(L.ss_decode_step, None, ctypes.byref(io), st) == B.SS_ERR_INVALID_ARG
    assert B.ss_get_phase(p) == (1, True)            # failed calls leave the plan unchanged
    with pytest.raises(B.SSError):
        B.ss_set_phase(p, 4, False)
    assert B.ss_launch_count() == 0


def test_state_map_config_sizes_and_traffic(L):
    """SS_COEF_STATE: the per-sequence map buffer, its validation and its bytes."""
    p = B.Plan(B.SS_GDN, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16, B.SS_COEF_STATE, 0.25)
    s = B.ss_buffer_sizes(p)
    assert s["coef_state"] == 3 * 12 * 128 * 2
    assert B.ss_buffer_sizes(B.Plan(B.SS_GDN, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16))["coef_state"] == 0
    fixed = B.Plan(B.SS_GDN, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16)
    d_s, d_f = B.ss_traffic_bytes(p, B.SS_OP_DECODE, 2), B.ss_traffic_bytes(fixed, B.SS_OP_DECODE, 2)
    # per-sequence maps replace the shared fp32 map read once per head
    assert d_s["read_bytes"] - d_f["read_bytes"] == 3 * 12 * 128 * 2 - 12 * 128 * 4
    f_s, f_f = B.ss_traffic_bytes(p, B.SS_OP_FLUSH), B.ss_traffic_bytes(fixed, B.SS_OP_FLUSH)
    assert f_s["write_bytes"] - f_f["write_bytes"] == 3 * 12 * 128 * 2
    assert f_s["paper_read_bytes"] == f_f["paper_read_bytes"]
    for mode, ridge in ((7, 0.0), (B.SS_COEF_STATE, -1.0), (B.SS_COEF_STATE, float("nan")),
                        (B.SS_COEF_STATE, float("inf"))):
        with pytest.raises(B.SSError) as e:
            B.Plan(B.SS_GDN, 1, 1, 64, 64, 4, [4], B.SS_F32, mode, ridge)
        assert e.value.status == B.SS_ERR_INVALID_ARG
    # the map needs U, per-warp partial sums and U^T U in the flush's tile buffer
    with pytest.raises(B.SSError) as e:
        B.Plan(B.SS_KDA, 1, 1, 64, 64, 4, [64], B.SS_F32, B.SS_COEF_STATE)
    assert e.value.status == B.SS_ERR_UNSUPPORTED
    for K, V in ((64, 64), (64, 128), (128, 64), (128, 128)):
        B.Plan(B.SS_MAMBA2, 1, 1, K, V, 16, [min(K, V) // 2], B.SS_BF16, B.SS_COEF_STATE)


def test_lrd_map_config_sizes_and_limits(L):
    """SS_COEF_LRD: the same map buffer and bytes as SS_COEF_STATE; its rank
    limit comes from its own scratch (pivots, diagonal, Gram matrix)."""
    lrd = B.Plan(B.SS_GDN, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16, B.SS_COEF_LRD, 0.25)
    st = B.Plan(B.SS_GDN, 3, 2, 128, 64, 6, [5, 7], B.SS_BF16, B.SS_COEF_STATE, 0.25)
    assert B.ss_buffer_sizes(lrd)["coef_state"] == B.ss_buffer_sizes(st)["coef_state"] == 3 * 12 * 128 * 2
    for op in (B.SS_OP_DECODE, B.SS_OP_FLUSH):
        assert B.ss_traffic_bytes(lrd, op, 2 if op == B.SS_OP_DECODE else 0) == \
            B.ss_traffic_bytes(st, op, 2 if op == B.SS_OP_DECODE else 0)
    for ridge in (-1.0, float("nan"), float("inf")):
        with pytest.raises(B.SSError) as e:
            B.Plan(B.SS_GDN, 1, 1, 64, 64, 4, [4], B.SS_F32, B.SS_COEF_LRD, ridge)
        assert e.value.status == B.SS_ERR_INVALID_ARG
    # largest ranks per shape: 56 (64 x 64), 64 (64 x 128), 81 (128 x 64), 118 (128 x 128)
    for (K, V), rmax in {(64, 64): 56, (64, 128): 64, (128, 64): 81, (128, 128): 118}.items():
        B.Plan(B.SS_KDA, 1, 1, K, V, 8, [rmax], B.SS_F32, B.SS_COEF_LRD)
        if rmax < K:
            with pytest.raises(B.SSError) as e:
                B.Plan(B.SS_KDA, 1, 1, K, V, 8, [rmax + 1], B.SS_F32, B.SS_COEF_LRD)
            assert e.value.status == B.SS_ERR_UNSUPPORTED


def test_dense_heads_config_and_traffic(L):
    """Dense-fallback heads: rank dk, their state copy in the sketch rows."""
    with pytest.raises(B.SSError) as e:
        B.Plan(B.SS_GDN, 2, 3, 128, 64, 8, [5, 64, 7], B.SS_BF16, dense_heads=[0, 1, 0])
    assert e.value.status == B.SS_ERR_INVALID_ARG and "dense head 1" in B.ss_last_error_string()
    d = B.Plan(B.SS_GDN, 2, 3, 128, 64, 8, [5, 128, 7], B.SS_BF16, dense_heads=[0, 1, 0])
    s = B.Plan(B.SS_GDN, 2, 3, 128, 64, 8, [5, 128, 7], B.SS_BF16)
    assert B.ss_buffer_sizes(d)["sketch"] == 2 * 140 * 64 * 2
    dd, ds = B.ss_traffic_bytes(d, B.SS_OP_DECODE, 3), B.ss_traffic_bytes(s, B.SS_OP_DECODE, 3)
    # the dense head's 128 basis/coef rows are not read
    assert ds["read_bytes"] - dd["read_bytes"] == 128 * 128 * 4
    fd, fs = B.ss_traffic_bytes(d, B.SS_OP_FLUSH), B.ss_traffic_bytes(s, B.SS_OP_FLUSH)
    # the copy re-reads each sequence's dense state once; no basis rows for it
    assert fd["read_bytes"] - fs["read_bytes"] == 2 * 128 * 64 * 4 - 128 * 128 * 4
    # paper metric: the dense head reads a bf16 state copy, dk x dv, per non-flush step
    assert dd["paper_read_bytes"] == 2 * (12 * (128 + 64) * 2 + 12 * 8 * 2 + 128 * 64 * 2)
    # a dense head does not raise the sketched heads' staging (rank 128 would not fit here)
    B.Plan(B.SS_KDA, 1, 2, 128, 128, 32, [128, 16], B.SS_F32, dense_heads=[1, 0])
    with pytest.raises(B.SSError):
        B.Plan(B.SS_KDA, 1, 2, 128, 128, 32, [128, 16], B.SS_F32)


@pytest.mark.skipif(not _no_gpu(), reason="fake-pointer validation tests run on CPU hosts only")
def test_state_map_needs_its_buffer(L):
    p = B.Plan(B.SS_KDA, 2, 2, 64, 64, 4, [2, 3], B.SS_F32, B.SS_COEF_STATE, 0.0)
    st = ctypes.c_void_p(0)
    io = _fake_io()
    B.ss_set_phase(p, 1, True)
    b = _fake_bufs(null="coef_state")
    assert L.ss_decode_step(p.handle, ctypes.byref(b), ctypes.byref(io), st) == B.SS_ERR_INVALID_ARG
    assert "coef_state" in B.ss_last_error_string()
    b = _fake_bufs(bad="coef_state")
    assert L.ss_decode_step(p.handle, ctypes.byref(b), ctypes.byref(io), st) == B.SS_ERR_ALIGNMENT
    B.ss_set_phase(p, 0, False)
    assert L.ss_prime(p.handle, ctypes.byref(_fake_bufs(null="coef_state")), st) == B.SS_ERR_INVALID_ARG
    B.ss_set_phase(p, 3, True)
    assert L.ss_flush(p.handle, ctypes.byref(_fake_bufs(null="coef_state")), ctypes.byref(io), st) == \
        B.SS_ERR_INVALID_ARG
    assert B.ss_launch_count() == 0


def _ratio(family, dk, dv, rank, W, heads=4, batch=3):
    p = B.Plan(family, batch, heads, dk, dv, W, [rank] * heads, B.SS_BF16)
    ex = B.ss_traffic_bytes(p, B.SS_OP_EXACT)
    std = ex["paper_read_bytes"] + ex["paper_write_bytes"]
    if rank == 0:   # ReplaySSM
        steps = [B.ss_traffic_bytes(p, B.SS_OP_REPLAY, t) for t in range(W - 1)]
        steps.append(B.ss_traffic_bytes(p, B.SS_OP_REPLAY_FLUSH))
    else:
        steps = [B.ss_traffic_bytes(p, B.SS_OP_DECODE, t) for t in range(W - 1)]
        steps.append(B.ss_traffic_bytes(p, B.SS_OP_FLUSH))
    per_step = sum(s["paper_read_bytes"] + s["paper_write_bytes"] for s in steps) / W
    return std / per_step


def test_traffic_model_reproduces_printed_reductions(L):
    with open(os.path.join(GOLDEN, "traffic_reduction.json")) as f:
        cases = json.load(f)["cases"]
    fam = {"mamba2": B.SS_MAMBA2, "gdn": B.SS_GDN, "kda": B.SS_KDA}
    for c in cases:
        got = _ratio(fam[c["family"]], c["dk"], c["dv"], c["rank"], c["window"])
        assert round(got, 2) == c["printed"], (c["name"], got)
    # KDA shares GDN's traffic model (same state and sketch sizes)
    assert round(_ratio(B.SS_KDA, 128, 128, 8, 16), 2) == 10.68
    assert abs(_ratio(B.SS_MAMBA2, 128, 64, 0, 16) - 32 / 17) < 1e-12


def test_all_bytes_model(L):
    """The roofline byte count: state, ring slots, inputs, sketch, basis, outputs."""
    K, V, W, Bt, H = 128, 64, 16, 5, 3
    p = B.Plan(B.SS_MAMBA2, Bt, H, K, V, W, [2, 8, 16], B.SS_BF16)
    R = 26
    slot = 2 * K + 2 * V + 4
    tok = 2 * K + slot
    dec = B.ss_traffic_bytes(p, B.SS_OP_DECODE, 7)
    assert dec["read_bytes"] == Bt * H * (tok + 7 * slot) + Bt * R * V * 2 + R * K * 4 + 4 * H
    assert dec["write_bytes"] == Bt * H * (slot + 4 * V)
    fl = B.ss_traffic_bytes(p, B.SS_OP_FLUSH)
    D = 4 * K * V
    assert fl["read_bytes"] == Bt * H * (D + (W - 1) * slot + tok) + R * K * 4 + 4 * H
    assert fl["write_bytes"] == Bt * H * (D + 4 * V) + Bt * R * V * 2
    with pytest.raises(B.SSError):
        B.ss_traffic_bytes(p, B.SS_OP_DECODE, W - 1)
    with pytest.raises(B.SSError):
        B.ss_traffic_bytes(p, 42)


def test_status_strings(L):
    assert B.ss_status_string(B.SS_ERR_SCHEDULE) == "SS_ERR_SCHEDULE"
    assert B.ss_status_string(99) == "unknown ss_status"


@pytest.mark.skipif(not _no_gpu(), reason="fake-pointer validation tests run on CPU hosts only")
def test_mixed_step_host_checks(L):
    """ss_step_mixed refuses bad fills and schedules before launching anything."""
    p = B.Plan(B.SS_GDN, 4, 2, 64, 64, 4, [2, 3])
    st = ctypes.c_void_p(0)
    bufs, io = _fake_bufs(), _fake_io()
    fin, fout = ctypes.c_void_p(0x700000), ctypes.c_void_p(0x710000)

    def rc(fi, fo, b=bufs):
        return L.ss_step_mixed(p.handle, ctypes.byref(b), ctypes.byref(io), fi, fo, st)

    assert rc(fin, fout) == B.SS_ERR_SCHEDULE                  # no sketch yet (ss_prime first)
    B.ss_set_phase(p, 2, True)
    assert rc(fin, fout) == B.SS_ERR_SCHEDULE                  # the plan must sit at phase 0
    B.ss_set_phase(p, 0, True)
    assert rc(None, fout) == B.SS_ERR_INVALID_ARG
    assert rc(fin, None) == B.SS_ERR_INVALID_ARG
    assert rc(ctypes.c_void_p(0x700002), fout) == B.SS_ERR_ALIGNMENT
    assert rc(fin, fin) == B.SS_ERR_INVALID_ARG                 # fill_out may not alias fill_in
    assert "alias" in B.ss_last_error_string()
    for name in ("sketch", "basis", "coef", "state"):
        assert rc(fin, fout, _fake_bufs(null=name)) == B.SS_ERR_INVALID_ARG, name
    assert B.ss_get_phase(p) == (0, True) and B.ss_launch_count() == 0
