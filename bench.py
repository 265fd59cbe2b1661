"""Throughput of the SketchSSM decode path on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--sketch-dtype bf16|f32] [--impl ours|reference]

A step is one decode window of the whole hot path over the workload's batch:
W-1 non-flush steps (ss_decode_step) and one flush (ss_flush), i.e. every
(sequence, head) advances W tokens.  The metric is decode steps per second in
(sequence x head) units: batch * heads * W per window / device time.

Timing: like a model's decode step, a step runs every layer of a stack of
--layers independent layers (own state, ring, sketch; default 4), so the
inputs of consecutive launches are far larger than L2 (126 MB) and nothing
is re-read from L2 across launches.  Launches go back to back; each is
bracketed by CUDA events on the launching stream for the per-kernel
figures, and the K timed windows by a barrier and torch.cuda.synchronize()
on both sides; the time is the max over ranks.  Under torchrun every rank decodes its own
copy of the workload (weak scaling; sequences are independent, so no data
collective exists on this path).

--impl reference times the fp64 CPU oracle on the host cores over a bounded
sample of the same workload (the pages publish no runnable implementation).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)


# ---------------------------------------------------------------------------
# distributed plumbing (barrier and max over ranks only)
# ---------------------------------------------------------------------------
def dist_init(backend):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    rank = dist.get_rank() if world > 1 else 0
    return rank, world


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: every rank processed units_per_rank in at most seconds_max."""
    return units_per_rank * world / seconds_max


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        t0 = time.time()                 # nvidia-smi takes a moment to print its first sample
        while time.time() - t0 < 10 and os.path.getsize(self.path) == 0:
            time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def kernel_source_sha():
    """Hash of the device-code sources (every CUDA source but the host-only
    API file), to tell whether ncu counters are still current."""
    d = os.path.join(ROOT, "ssm_decode_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f == "ss_api.cu":
            continue
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def kernel_traffic_record(name, workload, coef="fixed"):
    """ncu-measured DRAM bytes per launch, if taken on the current kernel source
    for this workload (the records are of the fixed-map mode)."""
    if coef != "fixed":
        return None
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        sha = kernel_source_sha()
        r = rec.get(f"{name}@{workload}") or rec.get(name)
        if r and r.get("source_sha") == sha and r.get("workload") == workload:
            return r
    except (OSError, ValueError):
        pass
    return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def sketch_vs_exact(layers, toks, W, torch):
    """Approximation metric of the sketched read: two layers start from the same
    state; one takes the window's non-flush steps through ss_decode_step
    (sketched read), the other through ss_replay_step (the exact windowed read
    S0^T q~ + buffered term, same library); their outputs are compared per
    (sequence, head): ||o^ - o||_2 / ||o||_2."""
    a, b = layers[0], layers[1]
    b.state.copy_(a.state)
    a.prime()
    b.prime()
    errs, nums, dens = [], 0.0, 0.0
    for p in range(W - 1):
        a.decode(toks[p])
        b.replay_step(toks[p])
        num = (a.out - b.out).double().norm(dim=-1)
        den = b.out.double().norm(dim=-1)
        errs.append((num / den.clamp_min(1e-300)).flatten())
        nums += float(num.sum())
        dens += float(den.sum())
    e = torch.cat(errs)
    res = {"metric": "sketch-vs-exact relative error ||o^ - o||_2 / ||o||_2 per (sequence, head) "
                      "over the non-flush steps of one window (sketched decode vs the exact replay read)",
            "mean": float(e.mean()), "p99": float(torch.quantile(e.float(), 0.99)), "max": float(e.max()),
            "aggregate": nums / max(dens, 1e-300),       # sum ||o^ - o|| / sum ||o||
            "outputs": int(e.numel())}
    # close the window so both layers are back at phase 0
    a.flush(toks[W - 1])
    b.replay_step(toks[W - 1])
    return res


def other_modes(args, wl, st, layers, toks, W, units, dev, stream, torch, B, DecodeLayer):
    """Outside the timed region: the same workload with sequences at mixed
    window positions (ss_step_mixed) and with the state-dependent map, each
    timed with CUDA events over a few steps.  Errors are reported, not raised."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    out = {}
    try:                                   # mixed positions: fills spread evenly over 0..W-1
        fills = [torch.arange(wl.batch, dtype=torch.int32, device=dev) % W for _ in layers]
        nxt = [torch.empty_like(f) for f in fills]
        ts = []
        for k in range(3):
            a, b = ev(), ev()
            a.record(stream)
            for p in range(W):
                for l, lay in enumerate(layers):
                    lay.step_mixed(toks[(p + l) % W], fills[l], nxt[l])
                    fills[l], nxt[l] = nxt[l], fills[l]
            b.record(stream)
            torch.cuda.synchronize()
            if k:
                ts.append(a.elapsed_time(b))
        ms = min(ts) / (W * len(layers))
        out["mixed"] = {"what": "ss_step_mixed, fills spread evenly over the window, every layer",
                        "us_per_step": ms * 1e3, "value": units / (ms / 1e3), "unit": "seq*heads/s",
                        "status": int(sum(int(l.status[0].item()) for l in layers))}
    except Exception as e:                 # noqa: BLE001 - reported in the line
        out["mixed"] = {"error": repr(e)[:200]}
    # the state-dependent coefficient maps (rho 0.01): the exact least-squares
    # map (paper §A.2.1) and the low-rank-plus-diagonal one (§A.2.2)
    for key, mode, what in (("state_map", B.SS_COEF_STATE, "the exact least-squares map"),
                            ("lrd_map", B.SS_COEF_LRD, "the low-rank-plus-diagonal map (4 pivots)")):
        try:
            import numpy as np  # noqa: F401
            skd = B.SS_BF16 if args.sketch_dtype == "bf16" else B.SS_F32
            sl = []
            for _ in range(2):
                lay = DecodeLayer(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, W, st.ranks, skd, device=dev,
                                  coef_mode=mode, coef_ridge=0.01)
                lay.state.copy_(layers[0].state)
                lay.basis.copy_(layers[0].basis)
                lay.A.copy_(layers[0].A)
                lay.prime()
                sl.append(lay)
            ts, fs = [], []
            for k in range(3):
                a, f0, b = ev(), ev(), ev()
                a.record(stream)
                for p in range(W):
                    if p == W - 1:
                        f0.record(stream)
                    for l, lay in enumerate(sl):
                        lay.step(toks[(p + l) % W])
                b.record(stream)
                torch.cuda.synchronize()
                if k:
                    ts.append(a.elapsed_time(b))
                    fs.append(f0.elapsed_time(b))
            ms = min(ts) / len(sl)
            approx = sketch_vs_exact(sl, toks, W, torch)
            out[key] = {"what": f"the same window with {what} (rho 0.01) built by every flush",
                        "ms_per_window": ms, "flush_us": min(fs) / len(sl) * 1e3,
                        "value": units * W / (ms / 1e3), "unit": "seq*heads/s",
                        "approx_mean": approx["mean"], "approx_aggregate": approx["aggregate"]}
            del sl
            torch.cuda.empty_cache()
        except Exception as e:             # noqa: BLE001
            out[key] = {"error": repr(e)[:200]}
    return out


NOMINAL_HBM_GBS = 8000.0        # B200 HBM3e data-sheet figure (context beside the measured copy peak)


def kernel_stats(plan, B, W, dec_ms, n_dec, fl_ms, n_fl, flush_name, peak, wl_name, coef="fixed"):
    """Per-kernel mean durations and HBM fractions: algorithmic bytes from the
    library's traffic model (mean over the window's decode positions for the
    decode) over the mean launch duration."""
    dec_bytes = [B.ss_traffic_bytes(plan, B.SS_OP_DECODE, p) for p in range(W - 1)]
    dec_b = sum(t["read_bytes"] + t["write_bytes"] for t in dec_bytes) / max(W - 1, 1)
    fl = B.ss_traffic_bytes(plan, B.SS_OP_FLUSH)
    fl_b = fl["read_bytes"] + fl["write_bytes"]
    kernel_ms = dec_ms + fl_ms
    kernels = {}
    for name, ms, count, nbytes in (("decode_kernel", dec_ms, n_dec, dec_b), (flush_name, fl_ms, n_fl, fl_b)):
        if not count:
            continue
        avg_s = ms / count / 1e3
        ach = nbytes / avg_s / 1e9
        rec = kernel_traffic_record(name, wl_name, coef)
        kernels[name] = {"launches": count, "avg_us": avg_s * 1e6, "bytes_per_launch": nbytes,
                         "achieved_gbs": ach, "frac": ach / peak, "frac_nominal": ach / NOMINAL_HBM_GBS,
                         "share": ms / kernel_ms,
                         "traffic": rec["dram_bytes_per_launch"] if rec else None,
                         "timing": "events at window boundaries and around the flush group"}
    return kernels


def flush_kernel_name(family, smap, synth, wl=None, rmax=0):
    """The kernel that runs a family's flush (see launch_flush in the library):
    Mamba-2 with the fixed map on the warp-MMA kernel; GDN and KDA with the
    fixed map, dv = 128, dk = 64 or 128, at most 16 updates and 32 read-out
    columns (rank + the token) on the tensor-core kernel; the rest on the
    CUDA-core kernel."""
    if family == synth.MAMBA2 and not smap:
        return "flush_mma_kernel"
    if (not smap and wl is not None and wl.dv == 128 and wl.dk in (64, 128) and wl.window <= 16
            and rmax + 1 <= 32):
        return "flush_tc_kernel"
    return "flush_kernel"


def other_families(args, dev, stream, torch, B, synth, DecodeLayer, peak, names=("gdn_b256", "kda_b256")):
    """Outside the timed region (rank 0): the GDN and KDA target workloads'
    decode and flush, timed like the headline workload (layers rotated so the
    inputs exceed L2, back-to-back launches, events at window boundaries), so
    one bench line carries every family's kernel fractions."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    out = {}
    for name in names:
        try:
            wl = synth.WORKLOADS[name]
            W, NL = wl.window, args.layers
            st = synth.static_inputs(wl)
            skd = B.SS_BF16 if args.sketch_dtype == "bf16" else B.SS_F32
            layers = []
            for _ in range(NL):
                lay = DecodeLayer(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, W, st.ranks, skd, device=dev)
                lay.load(st.state, st.basis, st.coef, st.A)
                layers.append(lay)
            toks = [layers[0].token(synth.step_inputs(wl, st, t)) for t in range(W)]
            for lay in layers:
                lay.prime()

            def window(marks=None):
                if marks:
                    marks[0].record(stream)
                for p in range(W):
                    if marks and p == W - 1:
                        marks[1].record(stream)
                    for l, lay in enumerate(layers):
                        lay.step(toks[(p + l) % W])
                if marks:
                    marks[2].record(stream)

            for _ in range(3):
                window()
            nwin = max(3, min(args.steps, 10))
            marks = [(ev(), ev(), ev()) for _ in range(nwin)]
            for m in marks:
                window(m)
            torch.cuda.synchronize()
            dec_ms = sum(m[0].elapsed_time(m[1]) for m in marks)
            fl_ms = sum(m[1].elapsed_time(m[2]) for m in marks)
            tot_ms = sum(m[0].elapsed_time(m[2]) for m in marks)
            kern = kernel_stats(layers[0].plan, B, W, dec_ms, nwin * NL * (W - 1), fl_ms, nwin * NL,
                                flush_kernel_name(wl.family, False, synth, wl, int(np.max(st.ranks))), peak,
                                wl.name)
            out[name] = {"value": wl.units * W * NL * nwin / (tot_ms / 1e3), "unit": "seq*heads/s",
                         "windows": nwin, "layers": NL, "kernels": kern,
                         "status": int(sum(int(l.status[0].item()) for l in layers))}
            del layers, toks
            torch.cuda.empty_cache()
        except Exception as e:             # noqa: BLE001 - reported in the line
            out[name] = {"error": repr(e)[:200]}
    return out


def run_ours(args, rank, world):
    import torch
    from ssm_decode_b200 import binding as B
    from ssm_decode_b200 import synth
    from ssm_decode_b200.layer import DecodeLayer

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[args.workload]
    if args.batch:
        wl = dataclasses.replace(wl, name=f"{wl.name}@batch{args.batch}", batch=args.batch)
    skd = B.SS_BF16 if args.sketch_dtype == "bf16" else B.SS_F32
    smap = args.coef in ("state", "lrd")
    W, NL = wl.window, args.layers
    st = synth.static_inputs(wl)
    layers = []
    for _ in range(NL):
        lay = DecodeLayer(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, W, st.ranks, skd, device=dev,
                          coef_mode={"state": B.SS_COEF_STATE, "lrd": B.SS_COEF_LRD}.get(args.coef, B.SS_COEF_FIXED),
                          coef_ridge=args.ridge)
        lay.load(st.state, st.basis, st.coef, st.A)
        layers.append(lay)
    st.state = None
    host_inputs = [synth.step_inputs(wl, st, t) for t in range(W)]
    toks = [layers[0].token(x) for x in host_inputs]
    stream = torch.cuda.current_stream()
    units = wl.units

    # One decode step of a model runs every layer; so does one step here.
    # Layer l at window position p reads token set (p + l) mod W, so a token
    # set is re-read only NL launches later, after far more than L2 (126 MB)
    # has streamed through.
    def ev():
        return torch.cuda.Event(enable_timing=True)

    def window(marks=None, call=lambda lay, tok: lay.step(tok), per_launch=None):
        # marks = (start, decodes done, end) events on the launching stream:
        # the window's decodes run between the first two, its flushes between
        # the last two.  per_launch[p][l] = an event pair around one launch
        # (a separate pass only: events between launches add gaps).
        if marks:
            marks[0].record(stream)
        for p in range(W):
            if marks and p == W - 1:
                marks[1].record(stream)
            for l, lay in enumerate(layers):
                if per_launch:
                    per_launch[p][l][0].record(stream)
                call(lay, toks[(p + l) % W])
                if per_launch:
                    per_launch[p][l][1].record(stream)
        if marks:
            marks[2].record(stream)

    for lay in layers:
        lay.prime()
    marks = [(ev(), ev(), ev()) for _ in range(args.steps)]
    # clocks are sampled from the start of the warm-up through the timed windows
    with ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        for _ in range(args.warmup):
            window()
        torch.cuda.synchronize()
        barrier(dev)
        n0 = B.ss_launch_count()
        t_all0, t_all1 = ev(), ev()
        torch.cuda.synchronize()
        t_all0.record(stream)
        for k in range(args.steps):
            window(marks[k])
        t_all1.record(stream)
        torch.cuda.synchronize()
        barrier(dev)
    launches = B.ss_launch_count() - n0
    dec_ms = sum(m[0].elapsed_time(m[1]) for m in marks)
    fl_ms = sum(m[1].elapsed_time(m[2]) for m in marks)
    n_dec, n_fl = args.steps * NL * (W - 1), args.steps * NL
    # per-position decode times, from a separate pass with events around each launch
    per_launch = [[(ev(), ev()) for _ in range(NL)] for _ in range(W)]
    window(per_launch=per_launch)
    torch.cuda.synchronize()
    total_ms = t_all0.elapsed_time(t_all1)
    total_ms_max = reduce_max(total_ms, dev)
    value = weak_scaling_value(units * W * NL * args.steps, world, total_ms_max / 1e3)

    # per-kernel roofline (algorithmic bytes from the library's traffic model)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    plan = layers[0].plan
    flush_name = flush_kernel_name(wl.family, smap, synth, wl, int(np.max(st.ranks)))
    kernels = kernel_stats(plan, B, W, dec_ms, n_dec, fl_ms, n_fl, flush_name, peak, wl.name, args.coef)
    if W > 1:
        kernels["decode_kernel"]["by_phase_us"] = [
            round(sum(per_launch[p][l][0].elapsed_time(per_launch[p][l][1]) for l in range(NL)) / NL * 1e3, 2)
            for p in range(W - 1)]
        kernels["decode_kernel"]["by_phase_note"] = "one extra window with events around each launch"
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    d = kernels[dom]
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(d["achieved_gbs"], 1), "peak": peak,
                "unit": "GB/s", "frac": round(d["frac"], 4), "traffic": d["traffic"],
                "peak_source": f"{peak_kind} hbm_gbs (burst copy; kernels timed inside the step)",
                "frac_nominal": round(d["achieved_gbs"] / NOMINAL_HBM_GBS, 4),
                "nominal_peak": NOMINAL_HBM_GBS}

    # baselines in the same library: Standard (exact step) and ReplaySSM
    baselines = {}
    for name, call in (("standard", lambda lay, tok: lay.exact_step(tok)),
                       ("replay", lambda lay, tok: lay.replay_step(tok))):
        ts = []
        for _ in range(2):
            a, b = ev(), ev()
            a.record(stream)
            window(call=call)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / NL)
        t = min(ts)
        baselines[name] = {"ms_per_window": t, "value": units * W / (t / 1e3),
                           "sketch_speedup": t / (total_ms / (args.steps * NL))}
    approx = sketch_vs_exact(layers, toks, W, torch) if NL >= 2 and W > 1 else None
    for lay in layers:
        lay.prime()

    # end to end through the C ABI: pinned host inputs in, outputs back, every
    # call.  Copies are pipelined the way a serving loop would run them: the
    # inputs of later launches are copied in on one stream and finished
    # outputs read back on another while the kernels run; NB device buffers
    # rotate, each copy waiting (CUDA events) for the last use of its buffer.
    keys = ("q", "k", "v", "gate") + (() if wl.family == synth.MAMBA2 else ("beta",))
    pin = [{k: torch.from_numpy(np.ascontiguousarray(x[k].view(np.int16) if x[k].dtype == np.uint16 else x[k]))
            .pin_memory() for k in keys} for x in host_inputs]
    host_out = torch.empty((W, NL) + tuple(layers[0].out.shape), dtype=torch.float32).pin_memory()
    h2d = NL * sum(t.numel() * t.element_size() for x in pin for t in x.values())
    d2h = host_out.numel() * host_out.element_size()
    NB = 2 * NL
    from ssm_decode_b200.layer import Token
    dev_tok = [Token({k: torch.empty_like(v) for k, v in toks[0].items()}) for _ in range(NB)]
    dev_out = [torch.empty_like(layers[0].out) for _ in range(NB)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    used = [None] * NB      # event: the kernel that last read dev_tok[i] / wrote dev_out[i] is done
    drained = [None] * NB   # event: dev_out[i] has been copied back
    e2e_times = []
    for k in range(args.warmup + args.steps):
        a, b = ev(), ev()
        torch.cuda.synchronize()
        a.record(stream)
        s_in.wait_event(a)
        s_out.wait_event(a)
        n = 0
        for p in range(W):
            for l, lay in enumerate(layers):
                i = n % NB
                with torch.cuda.stream(s_in):
                    if used[i] is not None:
                        s_in.wait_event(used[i])
                    for key, t in pin[(p + l) % W].items():
                        dev_tok[i][key].copy_(t, non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(s_in)
                stream.wait_event(ready)
                if drained[i] is not None:
                    stream.wait_event(drained[i])
                lay.step(dev_tok[i], out=dev_out[i])
                used[i] = torch.cuda.Event()
                used[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(used[i])
                    host_out[p, l].copy_(dev_out[i], non_blocking=True)
                    drained[i] = torch.cuda.Event()
                    drained[i].record(s_out)
                n += 1
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        b.record(stream)
        torch.cuda.synchronize()
        if k >= args.warmup:
            e2e_times.append(a.elapsed_time(b))
    e2e_ms = reduce_max(sum(e2e_times), dev)
    e2e = {"value": weak_scaling_value(units * W * NL * args.steps, world, e2e_ms / 1e3),
           "unit": "seq*heads/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "copies": "pinned host buffers; input copies and output read-backs pipelined on two "
                     "copy streams against the kernels, all inside the timed region"}

    modes = other_modes(args, wl, st, layers, toks, W, units, dev, stream, torch, B, DecodeLayer) \
        if rank == 0 else None
    del layers, toks, dev_tok, dev_out
    torch.cuda.empty_cache()
    families = None
    if rank == 0 and args.workload == "mamba2_b320" and not args.batch and not args.no_families:
        families = other_families(args, dev, stream, torch, B, synth, DecodeLayer, peak)

    result = {
        "metric": "decode steps/sec (seq*heads/s), flush + sketched decode",
        "value": value, "unit": "seq*heads/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "family": synth.FAMILY_NAMES[wl.family], "batch": wl.batch,
                   "heads": wl.heads, "dk": wl.dk, "dv": wl.dv, "window": W, "mean_rank": wl.mean_rank,
                   "layers": NL, "sketch": args.sketch_dtype, "inputs": "bf16 q/k/v, fp32 state",
                   "coef": ({"state": f"state-dependent map, rho = {args.ridge}",
                             "lrd": f"low-rank-plus-diagonal map, rho = {args.ridge}"}.get(args.coef, "fixed C = P^T")),
                   "step": f"one window of {W} tokens through {NL} independent layers",
                   "l2": f"inputs larger than L2: {NL} layers rotated, back-to-back launches",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline, "kernels": kernels, "baselines": baselines, "e2e": e2e,
        "gpu_launches": launches, "clocks": clk.summary(), "approx": approx, "modes": modes,
        "families": families,
    }
    return result


# ---------------------------------------------------------------------------
# the oracle on host cores (cpu_baseline, and the reference arm)
# ---------------------------------------------------------------------------
def oracle_window_rate(wl_name, n_seq, windows=1, budget_s=None):
    """Time the fp64 oracle decoding windows of a sample of n_seq sequences."""
    from threadpoolctl import threadpool_limits

    from oracle import sketchssm_oracle as orc
    from ssm_decode_b200 import synth
    wl = synth.WORKLOADS[wl_name]
    sub = synth.shrink(wl, batch=n_seq)
    st = synth.static_inputs(sub)
    inputs = [synth.step_inputs(sub, st, t) for t in range(wl.window)]
    sess = orc.Session(wl.family, st.state, wl.window, st.A, st.basis, st.coef, st.offsets,
                       sketch_bf16=True)
    with threadpool_limits(limits=1):
        sess.prime()
        times = []
        t_start = time.perf_counter()
        while True:
            t0 = time.perf_counter()
            for p in range(wl.window):
                sess.step(inputs[p])
            times.append(time.perf_counter() - t0)
            if budget_s is None and len(times) >= windows:
                break
            if budget_s is not None and time.perf_counter() - t_start >= budget_s:
                break
    units = n_seq * wl.heads * wl.window
    return units, times, wl


def _oracle_rate(wl_name, n_seq, budget_s):
    """One worker of the all-cores leg: the oracle's rate on its own copy of the
    sample.  Its input generation runs single-threaded too: one BLAS thread pool
    per core-sized process would oversubscribe the host many times over."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        units, times, _ = oracle_window_rate(wl_name, n_seq, budget_s=budget_s)
    return units * len(times) / sum(times), len(times)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


MAX_ORACLE_WORKERS = 32          # bounds the leg's memory on large hosts


def cpu_baseline(args, one_s=12.0, each_s=10.0, max_workers=MAX_ORACLE_WORKERS, timeout_s=180.0):
    """The oracle on the host cores: one thread, then one single-threaded
    process per core (spawned, so none inherits the CUDA context), each
    decoding its own copy of the sample for a fixed time; the value is the sum
    of their rates.  Any failure of the parallel leg leaves the 1-thread figure."""
    n_seq = 4
    units, times, wl = oracle_window_rate(args.workload, n_seq, budget_s=one_s)
    one = units / (sum(times) / len(times))
    sample = (f"{n_seq} of {wl.batch} sequences x {wl.heads} heads, full windows of {wl.window} steps, "
              f"fp64 numpy, single-threaded per process")
    res = {"value": one, "unit": "seq*heads/s", "cores": 1, "kind": "oracle",
           "sample": f"{sample}; 1 thread, {len(times)} windows",
           "one_thread": {"value": one, "windows": len(times)}}
    workers = min(host_cores(), max_workers)
    if workers > 1:
        import multiprocessing as mp
        try:
            with mp.get_context("spawn").Pool(workers) as pool:
                out = pool.starmap_async(_oracle_rate, [(args.workload, n_seq, each_s)] * workers).get(timeout=timeout_s)
            res["value"] = sum(r for r, _ in out)
            res["cores"] = workers
            res["sample"] = (f"{sample}; {workers} processes x {each_s:g} s each "
                             f"({min(w for _, w in out)}-{max(w for _, w in out)} windows per process)")
        except Exception as e:                      # noqa: BLE001 -- report the 1-thread figure
            res["parallel_error"] = f"{type(e).__name__}: {e}"[:200]
    return res


def run_reference(args):
    n_seq = 2
    units, times, wl = oracle_window_rate(args.workload, n_seq, windows=args.warmup + args.steps)
    times = times[args.warmup:] or times
    t = sum(times)
    value = units * len(times) / t
    return {
        "metric": "decode steps/sec (seq*heads/s), flush + sketched decode", "impl": "reference",
        "value": value, "unit": "seq*heads/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t / len(times) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "dk": wl.dk, "dv": wl.dv,
                   "window": wl.window, "mean_rank": wl.mean_rank, "sketch": "bf16"},
        "cpu_baseline": {"value": value, "unit": "seq*heads/s", "cores": 1, "kind": "oracle",
                         "sample": f"{n_seq} of {wl.batch} sequences x {wl.heads} heads per step "
                                   f"(one window of {wl.window} tokens), fp64 numpy, 1 thread"},
        "e2e": {"value": value, "unit": "seq*heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_sweep(args):
    """The sweep on the Mamba-2 shape: batch x window x mean rank, sketched
    flush + decode against the Standard and ReplaySSM steps of the same
    library, with the decode / flush HBM GB/s and the sketch-vs-exact error.
    One JSON line per point, then a markdown table."""
    import torch
    from ssm_decode_b200 import binding as B
    from ssm_decode_b200 import synth
    from ssm_decode_b200.layer import DecodeLayer

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peak = float(measured_peaks()[0]["hbm_gbs"])
    rows = []
    batches = [int(x) for x in args.sweep_batches.split(",")]
    windows = [int(x) for x in args.sweep_windows.split(",")]
    ranks = [int(x) for x in args.sweep_ranks.split(",")]
    for batch in batches:
        for W in windows:
            for mr in ranks:
                wl = synth.sweep_workload(batch, W, mr)
                st = synth.static_inputs(wl)
                # enough layers that the rotated inputs exceed L2 (126 MB), at least 2
                per_layer = wl.units * wl.dk * wl.dv * 4
                NL = max(2, min(8, -(-400_000_000 // per_layer)))
                layers = []
                for _ in range(NL):
                    lay = DecodeLayer(wl.family, wl.batch, wl.heads, wl.dk, wl.dv, W, st.ranks, B.SS_BF16, device=dev)
                    lay.load(st.state, st.basis, st.coef, st.A)
                    layers.append(lay)
                toks = [layers[0].token(synth.step_inputs(wl, st, t)) for t in range(W)]
                for lay in layers:
                    lay.prime()

                def run(call, marks=None):
                    if marks:
                        marks[0].record(stream)
                    for p in range(W):
                        if marks and p == W - 1:
                            marks[1].record(stream)
                        for l, lay in enumerate(layers):
                            call(lay, toks[(p + l) % W])
                    if marks:
                        marks[2].record(stream)

                ev = lambda: torch.cuda.Event(enable_timing=True)
                res = {}
                for name, call in (("sketch", lambda lay, tok: lay.step(tok)),
                                   ("standard", lambda lay, tok: lay.exact_step(tok)),
                                   ("replay", lambda lay, tok: lay.replay_step(tok))):
                    run(call)                                  # warm-up window
                    ms = []
                    for _ in range(args.sweep_windows_timed):
                        m = (ev(), ev(), ev())
                        run(call, m)
                        torch.cuda.synchronize()
                        ms.append((m[0].elapsed_time(m[2]), m[0].elapsed_time(m[1]), m[1].elapsed_time(m[2])))
                    best = min(ms)
                    res[name] = best
                    if name != "sketch":
                        for lay in layers:
                            lay.prime()
                t_win, t_dec, t_fl = res["sketch"]
                plan = layers[0].plan
                dec_b = (sum(sum(B.ss_traffic_bytes(plan, B.SS_OP_DECODE, p)[k] for k in ("read_bytes", "write_bytes"))
                             for p in range(W - 1)) / max(W - 1, 1))
                fl = B.ss_traffic_bytes(plan, B.SS_OP_FLUSH)
                fl_b = fl["read_bytes"] + fl["write_bytes"]
                dec_us = t_dec / max(NL * (W - 1), 1) * 1e3
                fl_us = t_fl / NL * 1e3
                approx = sketch_vs_exact(layers, toks, W, torch) if W > 1 else None
                row = {"batch": batch, "window": W, "mean_rank": mr, "layers": NL,
                       "sketch_steps_per_s": wl.units * W * NL / (t_win / 1e3),
                       "standard_steps_per_s": wl.units * W * NL / (res["standard"][0] / 1e3),
                       "replay_steps_per_s": wl.units * W * NL / (res["replay"][0] / 1e3),
                       "decode_us": dec_us, "decode_gbs": dec_b / (dec_us * 1e-6) / 1e9 if W > 1 else None,
                       "flush_us": fl_us, "flush_gbs": fl_b / (fl_us * 1e-6) / 1e9,
                       "err_mean": approx["mean"] if approx else 0.0, "err_max": approx["max"] if approx else 0.0}
                rows.append(row)
                print(json.dumps(row), flush=True)
                del layers, toks
                torch.cuda.empty_cache()
    print("| batch | W | mean r | sketch steps/s | vs Standard | vs Replay | decode µs (GB/s) | flush µs (GB/s) | "
          "sketch-vs-exact err mean / max |")
    print("|---|---|---|---|---|---|---|---|---|")
    for r in rows:
        dec = f"{r['decode_us']:.1f} ({r['decode_gbs']:.0f})" if r["decode_gbs"] else "-"
        print(f"| {r['batch']} | {r['window']} | {r['mean_rank']} | {r['sketch_steps_per_s']:.3g} | "
              f"{r['sketch_steps_per_s'] / r['standard_steps_per_s']:.2f}x | "
              f"{r['sketch_steps_per_s'] / r['replay_steps_per_s']:.2f}x | {dec} | "
              f"{r['flush_us']:.1f} ({r['flush_gbs']:.0f}) | {r['err_mean']:.3g} / {r['err_max']:.3g} |")
    print(f"(peak: measured {peak:.0f} GB/s)")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="mamba2_b320")
    ap.add_argument("--sketch-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-families", action="store_true",
                    help="skip the GDN / KDA kernel timings that follow the default Mamba-2 line")
    ap.add_argument("--coef", default="fixed", choices=["fixed", "state", "lrd"],
                    help="coefficient map: the fixed C = P^T of the workloads, the state-dependent "
                         "least-squares map rebuilt by every flush, or its low-rank-plus-diagonal form")
    ap.add_argument("--ridge", type=float, default=0.01, help="rho of the state-dependent maps")
    ap.add_argument("--sweep", action="store_true",
                    help="the batch x window x rank sweep on the Mamba-2 shape (1 GPU), instead of the bench line")
    ap.add_argument("--sweep-batches", default="1,32,128,320,1024")
    ap.add_argument("--sweep-windows", default="4,8,16,32")
    ap.add_argument("--sweep-ranks", default="4,8,16")
    ap.add_argument("--sweep-windows-timed", type=int, default=3)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.sweep:
        run_sweep(args)
        return

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    rank, world = dist_init("nccl")
    res = run_ours(args, rank, world)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args)
        print(json.dumps(res), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
