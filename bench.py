"""Benchmark of the BitLinear forward on the five workloads.

Headline (the JSON line's `value`): the 125M-shape decode workload.  One
step = the decode hot path for every projection of all 12 layers (q,o
768x768; k,v 256x768; gate,up 2048x768; down 768x2048 -- 84 problems) at
M = 1, 4 and 8 tokens: per M, ONE grouped launch that quantizes the bf16
activations, runs the ternary GEMV and rescales (bl_linear_decode_grouped).
The ternary weights (29/42/29 split) are packed once at load time.  Weight
bytes per step would fit in L2, so the packed weights are replicated and
every launch reads a different replica than the launches around it (the
replicas total more than 3x the L2 size).  Metric: decode GB/s = (packed
weight bytes + bf16 activation bytes) per step / time, whole job, N GPUs =
N independent replicas of the workload (weak scaling).

Every timed region runs exactly --steps steps between a barrier and a
device synchronization on both sides; the region is repeated (at least 20
times and --min-timed-ms of timed work in all) and the median is reported,
with the spread.

The other workloads are reported under "configs", each with its own
throughput, roofline, clock record, CPU-oracle baseline and end-to-end
figure through the C ABI with host buffers:
  single      one BitLinear 768 -> 2048, M = 16, fp32 W and X: the whole
              call (bl_linear) and each of its steps
  prefill1b4  the 1.4B-shape layer at M = 8192: the engine on pre-quantized
              inputs and the per-call path (weights quantized every call)
  layer3b     the 3B-shape layer: decode M = 1 (HBM) and prefill M = 2048
  qat4b       the 4B-shape QAT layer at M = 32768: per-call path with SubLN
              before o_proj and down_proj

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--only name,name] [--no-cpu-baseline] [--no-e2e]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from ternary_quantized_linear_bitlinear_b200 import workloads  # noqa: E402

METRIC = "BitLinear decode weight GB/s & prefill int8 TOPS, as % of roofline"
UNIT = "GB/s"
MS = (1, 4, 8)
SPAD = {M: (M + 3) // 4 * 4 for M in MS}
WORKLOAD = "decode125m: 12 layers x {q,o 768x768; k,v 256x768; gate,up 2048x768; down 768x2048}, M in {1,4,8}"
CONFIGS = ("single", "decode125m", "prefill1b4", "layer3b", "qat4b")
PER_CALL = ("per_call", "per_call_grouped", "per_call_layer")  # per-call paths of the prefill workloads


def replica_of(step: int, j: int, replicas: int) -> int:
    """Weight replica read by launch j (the j-th M) of a step: consecutive
    launches never share weights (the launches of one step included), so no
    launch is fed from L2; a replica comes back every `replicas` launches."""
    return (len(MS) * step + j) % replicas


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-alt", action="store_true", help="skip the secondary decode paths (per-M, two-launch, chains)")
    ap.add_argument("--min-timed-ms", type=float, default=300.0,
                    help="each measurement repeats its timed region until this much device time is timed")
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="reference arm: seconds of oracle work over the whole run")
    ap.add_argument("--only", default=",".join(CONFIGS),
                    help="comma-separated workloads to measure (decode125m is the headline)")
    return ap.parse_args(argv)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(xs, world: int):
    """Elementwise max over ranks of a list of floats (or of one float)."""
    single = not isinstance(xs, (list, tuple))
    vals = [xs] if single else list(xs)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor(vals, dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        vals = t.tolist()
    return vals[0] if single else vals


def peaks():
    """Roofline denominators: the measured peaks when present, else
    this pool's earlier measurement (the fallback)."""
    try:
        p = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        p = {}
    hbm = p.get("hbm_gbs")
    bf16 = p.get("bf16_tflops")
    bf16s = p.get("bf16_tflops_sustained")
    return {
        "hbm": float(hbm) if hbm else 6650.0,
        "hbm_source": "measured" if hbm else "fallback",
        # dense int8 = the bf16 figure x the nominal int8 : bf16 ratio (4.5 : 2.25)
        "int8": 2.0 * float(bf16) if bf16 else 2.0 * 1590.0,
        "int8_sustained": 2.0 * float(bf16s) if bf16s else 2.0 * 1400.0,
        "int8_source": ("measured bf16 x 2 (nominal int8:bf16)" if bf16 else "fallback bf16 x 2 (nominal int8:bf16)"),
    }


class Clocks:
    """nvidia-smi sampling during a timed region."""

    def __init__(self, index: int, tag: str = ""):
        self.index = str(index)
        try:
            uuid = torch.cuda.get_device_properties(index).uuid
            self.index = f"GPU-{uuid}"
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                self.index = vis.split(",")[index]
        self.proc = None
        # the raw samples go to $BL_CLOCKS_DIR (default: the temp directory)
        self.path = os.path.join(os.environ.get("BL_CLOCKS_DIR") or tempfile.gettempdir(),
                                 f"clocks_rank{index}{'_' + tag if tag else ''}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
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
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples under load: the power draw separates them from the idle gaps
        pmax = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, _, r in load for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(load), "power_w_median": round(statistics.median(r[2] for r in load), 1)}


def time_regions(run_once, stream, world, min_reps=20, min_ms=300.0, max_reps=2000):
    """Times `run_once()` (work enqueued on `stream`) as a repeated region:
    barrier + synchronize, event, work, event, synchronize, on every rank;
    repeated at least `min_reps` times and until `min_ms` of device time has
    been timed.  Returns the per-region times in ms (max over ranks)."""
    out = []
    total = 0.0
    while len(out) < min_reps or (total < min_ms and len(out) < max_reps):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            run_once()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        out.append(ms)
        total += ms
    barrier(world)
    return max_over_ranks(out, world)


def spread(ms):
    s = sorted(ms)
    return {"median_ms": round(statistics.median(s), 6), "min_ms": round(s[0], 6), "max_ms": round(s[-1], 6),
            "regions": len(s)}


def graph_of(fn, stream, warm=1):
    """fn(stream_ptr) enqueues work; returns a CUDA graph of one call (after
    `warm` eager calls, which also run the library's one-time set-up)."""
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn(sp)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(stream.cuda_stream)
    torch.cuda.synchronize()
    return g


def ok(rc, what):
    if rc:
        from ternary_quantized_linear_bitlinear_b200 import api
        raise api.BitLinearError(rc, what)


def roofline_hbm(kernel, bytes_per_launch, us_per_launch, pk, traffic=None, note=None):
    achieved = bytes_per_launch / (us_per_launch * 1e-6) / 1e9
    r = {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": pk["hbm"],
         "peak_source": pk["hbm_source"], "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4),
         "traffic": traffic, "avg_launch_us": round(us_per_launch, 3),
         "algorithmic_bytes_per_launch": int(bytes_per_launch)}
    if note:
        r["note"] = note
    return r


def roofline_tensor(kernel, ops, ms, pk, measured_on):
    tops = ops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": kernel, "measured_on": measured_on, "achieved": round(tops, 1),
            "peak": round(pk["int8"], 1), "unit": "TOPS", "peak_source": pk["int8_source"],
            "frac": round(tops / pk["int8"], 4), "frac_of_sustained": round(tops / pk["int8_sustained"], 4),
            "traffic": None}


def decode_traffic():
    """DRAM bytes per grouped decode launch from the committed ncu capture, or
    None when the kernel source changed since the counters were taken."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "decode_traffic.json")))
        src = open(os.path.join(ROOT, rec["kernel_source"]), "rb").read()
    except (OSError, ValueError, KeyError):
        return None
    if hashlib.sha256(src).hexdigest() != rec.get("kernel_source_sha256"):
        return None
    return rec.get("dram_bytes_per_launch")


def pinned(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().pin_memory()


class E2E:
    """Steps through the C ABI with host buffers: each step uploads its inputs
    from pinned host memory, runs, and downloads its outputs; `slots` device
    buffer sets and three streams (upload, compute, download) let one step's
    copies overlap another step's kernels, as a serving loop would.  Returns
    seconds per step (wall clock over `steps` steps, max over ranks)."""

    def __init__(self, dev, host_in, dev_in_slots, dev_out_slots, host_out_slots, compute, stream):
        self.dev = dev
        self.host_in = host_in              # list of pinned host tensors
        self.dev_in = dev_in_slots          # [slot][i] device tensors, same shapes
        self.dev_out = dev_out_slots        # [slot][j]
        self.host_out = host_out_slots      # [slot][j] pinned host tensors
        self.compute = compute              # compute(slot, step, stream_ptr)
        self.stream = stream

    def _step(self, it, s_up, s_dn, ev_up, ev_comp, ev_dn):
        k = it % len(self.dev_in)
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_comp[k])          # the kernels that read this slot's inputs are done
            for h, d in zip(self.host_in, self.dev_in[k]):
                d.copy_(h, non_blocking=True)
            ev_up[k].record(s_up)
        self.stream.wait_event(ev_up[k])
        self.stream.wait_event(ev_dn[k])         # this slot's previous outputs have been read back
        self.compute(k, it, self.stream.cuda_stream)
        ev_comp[k].record(self.stream)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev_comp[k])
            for d, h in zip(self.dev_out[k], self.host_out[k]):
                h.copy_(d, non_blocking=True)
            ev_dn[k].record(s_dn)

    def run_graph(self, steps_per_graph, replays, world):
        """The same loop captured once as a CUDA graph over the three streams
        (uploads, kernels and downloads all inside it; a serving loop would
        replay it), then replayed: seconds per step, wall clock over the
        replays (max over ranks)."""
        slots = len(self.dev_in)
        s_up = torch.cuda.Stream(device=self.dev)
        s_dn = torch.cuda.Stream(device=self.dev)
        ev_up = [torch.cuda.Event() for _ in range(slots)]
        ev_comp = [torch.cuda.Event() for _ in range(slots)]
        ev_dn = [torch.cuda.Event() for _ in range(slots)]
        for it in range(2):  # eager warm-up (the library's one-time set-up)
            self._step(it, s_up, s_dn, ev_up, ev_comp, ev_dn)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            fork = torch.cuda.Event()
            fork.record(self.stream)
            s_up.wait_event(fork)
            s_dn.wait_event(fork)
            for k in range(slots):  # the slots start free inside the graph
                ev_comp[k].record(self.stream)
                ev_dn[k].record(self.stream)
            for it in range(steps_per_graph):
                self._step(it, s_up, s_dn, ev_up, ev_comp, ev_dn)
            join_u, join_d = torch.cuda.Event(), torch.cuda.Event()
            join_u.record(s_up)
            join_d.record(s_dn)
            self.stream.wait_event(join_u)
            self.stream.wait_event(join_d)
        g.replay()
        torch.cuda.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        for _ in range(replays):
            g.replay()
        torch.cuda.synchronize()
        secs = time.perf_counter() - t0
        barrier(world)
        del g
        return max_over_ranks(secs, world) / (replays * steps_per_graph)

    def run(self, steps, world, warm=2):
        slots = len(self.dev_in)
        s_up = torch.cuda.Stream(device=self.dev)
        s_dn = torch.cuda.Stream(device=self.dev)
        ev_up = [torch.cuda.Event() for _ in range(slots)]
        ev_comp = [torch.cuda.Event() for _ in range(slots)]
        ev_dn = [torch.cuda.Event() for _ in range(slots)]
        sp = self.stream.cuda_stream
        torch.cuda.synchronize()
        barrier(world)
        t0 = None
        for it in range(steps + warm):
            if it == warm:
                torch.cuda.synchronize()
                barrier(world)
                t0 = time.perf_counter()
            k = it % slots
            with torch.cuda.stream(s_up):
                s_up.wait_event(ev_comp[k])          # the kernels that read this slot's inputs are done
                for h, d in zip(self.host_in, self.dev_in[k]):
                    d.copy_(h, non_blocking=True)
                ev_up[k].record(s_up)
            self.stream.wait_event(ev_up[k])
            self.stream.wait_event(ev_dn[k])         # this slot's previous outputs have been read back
            self.compute(k, it, sp)
            ev_comp[k].record(self.stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(ev_comp[k])
                for d, h in zip(self.dev_out[k], self.host_out[k]):
                    h.copy_(d, non_blocking=True)
                ev_dn[k].record(s_dn)
        torch.cuda.synchronize()
        secs = time.perf_counter() - t0
        barrier(world)
        return max_over_ranks(secs, world) / steps


def nbytes(ts):
    return sum(t.numel() * t.element_size() for t in ts)


# =============================================================================
# Headline: the 125M decode workload


def step_bytes():
    """Algorithmic bytes of one step: packed weights + x_q, per M."""
    shapes = workloads.decode125m_layer_shapes()
    L = workloads.DECODE125M["layers"]
    wbytes = L * sum(N * K // 4 for _, N, K, _ in shapes)
    xbytes = {M: L * sum(M * K for _, N, K, _ in shapes) for M in MS}
    return wbytes, xbytes


def bench_decode125m(args, rank, world, local, dev, pk):
    from ternary_quantized_linear_bitlinear_b200 import api

    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    wbytes, xbytes = step_bytes()
    R = max(2, (3 * l2) // wbytes + 1)  # weight replicas totalling > 3x L2

    # ---- load: pack the ternary weights once per replica (not timed) -------
    items = workloads.decode125m(seed=1 + rank, M=max(MS))
    shapes = [(W.shape[0], W.shape[1]) for _, W, _ in items]
    packed0, gammas = [], []
    for _, W, _ in items:
        p, g = api.bl_quant_weights(W.to(dev))
        packed0.append(p)
        gammas.append(g)
    flat0 = torch.cat([p.view(-1) for p in packed0])
    offs, o = [], 0
    for p in packed0:
        offs.append(o)
        o += p.numel()
    replicas = [flat0] + [flat0.clone() for _ in range(R - 1)]

    # activations: per M, views into ONE input buffer and ONE output buffer
    # for the whole step (so the end-to-end run moves each step's data in one
    # copy per direction)
    xlen = {M: sum(M * K for _, K in shapes) for M in MS}                  # multiples of 64: 128-byte aligned views
    ylen = {M: sum(M * N for N, _ in shapes) + 4 * len(items) for M in MS}  # per-problem slots padded to 4
    x_all_host = torch.cat([torch.cat([X[:M].contiguous().view(-1) for _, _, X in items]) for M in MS]).pin_memory()
    x_all = x_all_host.to(dev)
    y_all = torch.empty(sum(ylen.values()), dtype=torch.float32, device=dev)
    y_all_host = torch.empty_like(y_all, device="cpu").pin_memory()

    def split(buf, lens):
        out, o = {}, 0
        for M in MS:
            out[M] = buf[o:o + lens[M]]
            o += lens[M]
        return out

    xin, Y = split(x_all, xlen), split(y_all, ylen)
    xq = {M: torch.empty(xlen[M], dtype=torch.int8, device=dev) for M in MS}       # two-launch path only
    sc = {M: torch.empty(len(items) * SPAD[M], dtype=torch.float32, device=dev) for M in MS}

    def views(M, xbuf, ybuf):
        out, xo, yo = [], 0, 0
        for i, (N, K) in enumerate(shapes):
            out.append((xbuf[M][xo:xo + M * K], xq[M][xo:xo + M * K], sc[M][i * SPAD[M]:i * SPAD[M] + M],
                        ybuf[M][yo:yo + M * N], N, K))
            xo += M * K
            yo += (M * N + 3) // 4 * 4
        return out

    def fused_problems(M, rep, sel=None, xbuf=None, ybuf=None):
        v = views(M, xin if xbuf is None else xbuf, Y if ybuf is None else ybuf)
        idx = range(len(v)) if sel is None else sel
        arr = (api.DecodeProblem * len(idx))()
        base = replicas[rep].data_ptr()
        for j, i in enumerate(idx):
            X, _, _, y, N, K = v[i]
            arr[j] = api.DecodeProblem(base + offs[i], gammas[i].data_ptr(), X.data_ptr(), None, y.data_ptr(), None,
                                       None, None, N, K)
        return arr

    def two_launch_problems(M, rep):
        v = views(M, xin, Y)
        acts = (api.ActProblem * len(v))()
        fwd = (api.Problem * len(v))()
        base = replicas[rep].data_ptr()
        for i, (X, q, s_, y, N, K) in enumerate(v):
            acts[i] = api.ActProblem(X.data_ptr(), None, q.data_ptr(), s_.data_ptr(), K)
            fwd[i] = api.Problem(base + offs[i], gammas[i].data_ptr(), q.data_ptr(), s_.data_ptr(), y.data_ptr(), None,
                                 N, K)
        return acts, fwd

    L = api.lib()
    count = len(items)
    fused = {(M, r): fused_problems(M, r) for M in MS for r in range(R)}
    RDY = api.BL_FWD_WEIGHTS_READY
    stream = torch.cuda.Stream(device=dev)
    K_ = max(1, args.steps)

    def steps_fn(nsteps, ms=MS):
        def fn(sp):
            for st in range(nsteps):
                for j, M in enumerate(ms):
                    ok(L.bl_linear_decode_grouped(fused[(M, replica_of(st, MS.index(M), R))], count, api.BL_BF16,
                                                  M, 1e-6, RDY, sp), "bl_linear_decode_grouped")
        return fn

    # ---- exactly K steps per timed region, as one CUDA graph ---------------
    g_step = graph_of(steps_fn(K_), stream)
    for _ in range(max(1, math.ceil(max(3, args.warmup) / K_))):
        with torch.cuda.stream(stream):
            g_step.replay()
    torch.cuda.synchronize()
    with Clocks(local, "decode125m") as clk:
        ms = time_regions(g_step.replay, stream, world, min_ms=args.min_timed_ms)
    api.bl_check_device_error(stream)
    med = statistics.median(ms)
    bytes_step = sum(wbytes + 2 * xbytes[M] for M in MS)  # packed W + bf16 X read by the fused kernel
    value = world * bytes_step * K_ / (med * 1e-3) / 1e9
    dec_us = med * 1e3 / (K_ * len(MS))
    roof = roofline_hbm("k_decode (fused act quant + ternary GEMV + rescale, 84 problems)", bytes_step / len(MS),
                        dec_us, pk, decode_traffic())

    # per M: K launches of that M alone
    per_m = {}
    for M in (() if args.no_alt else MS):
        g = graph_of(steps_fn(K_, (M,)), stream)
        msm = time_regions(g.replay, stream, world, min_ms=args.min_timed_ms / 3)
        us = statistics.median(msm) * 1e3 / K_
        b = wbytes + 2 * xbytes[M]
        per_m[f"M={M}"] = {"us_per_launch": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                           "frac": round(b / (us * 1e-6) / 1e9 / pk["hbm"], 4)}
        del g
    roof["per_m"] = per_m

    # ---- secondary: two launches per M; layer order at M = 1 ---------------
    alt = {}
    nalt = max(1, min(K_, 2 * R))
    if args.no_alt:
        nalt = 0
    tl = {(M, r): two_launch_problems(M, r) for M in MS for r in range(R)}

    def two_step(sp):
        for st in range(nalt):
            for j, M in enumerate(MS):
                acts, fwd = tl[(M, replica_of(st, j, R))]
                ok(L.bl_quant_act_grouped(acts, count, api.BL_BF16, M, 1e-6, sp), "bl_quant_act_grouped")
                ok(L.bl_forward_grouped(fwd, count, M, RDY, sp), "bl_forward_grouped")

    if nalt:
        g2 = graph_of(two_step, stream)
        alt["two_launch_us_per_step"] = round(statistics.median(time_regions(g2.replay, stream, world, min_reps=10,
                                                                             min_ms=50)) * 1e3 / nalt, 3)
        del g2
    # the real dependent step: each layer reads the previous layer's output
    # (chain.DecodeChain), one chain per weight replica so that no step finds
    # its weights in L2
    from ternary_quantized_linear_bitlinear_b200.chain import PROJ, DecodeChain
    per_layer = len(PROJ)
    nlay = count // per_layer
    gains = [(workloads.uniform((768,), 0.9, 1.1, 30 + li).to(dev), workloads.uniform((2048,), 0.9, 1.1, 60 + li).to(dev))
             for li in range(nlay)]
    for Mc in ((1, 4) if nalt else ()):
        chains = []
        for r in range(R):
            layers = []
            for li in range(nlay):
                lay = {}
                for j, name in enumerate(PROJ):
                    i = li * per_layer + j
                    N, K = shapes[i]
                    lay[name] = (replicas[r][offs[i]:offs[i] + N * K // 4].view(N, K // 4), gammas[i], N, K)
                layers.append(lay)
            ch = DecodeChain(layers, gains, Mc)
            ch.x0.copy_(items[0][2][:Mc].float().to(dev))
            chains.append(ch)

        def chained(sp, chains=chains):
            for st in range(nalt):
                chains[st % R].run(sp)

        g3 = graph_of(chained, stream)
        us3 = statistics.median(time_regions(g3.replay, stream, world, min_reps=10, min_ms=50)) * 1e3 / nalt
        abytes = wbytes + 4 * Mc * sum(K for _, K in shapes)  # packed W + the f32 activations each layer reads
        alt[f"chain_m{Mc}"] = {"us_per_token_step": round(us3, 3), "gbs": round(abytes / (us3 * 1e-6) / 1e9, 1),
                               "launches_per_step": chains[0].launches_per_step(),
                               "note": "12 dependent layers: qkv | o (SubLN) | gate,up | FFN act quant (SubLN) "
                                       "| down, each reading the previous launch's output"}
        del g3, chains
    api.bl_check_device_error(stream)

    # ---- end to end through the C ABI with host buffers --------------------
    e2e = None
    if not args.no_e2e:
        slots = 2
        xa = [x_all] + [torch.empty_like(x_all) for _ in range(slots - 1)]
        ya = [y_all] + [torch.empty_like(y_all) for _ in range(slots - 1)]
        yah = [y_all_host] + [torch.empty_like(y_all_host).pin_memory() for _ in range(slots - 1)]
        xs = [split(b, xlen) for b in xa]
        ys = [split(b, ylen) for b in ya]
        slot_arrs = [{(M, r): fused_problems(M, r, None, xs[k], ys[k]) for M in MS for r in range(R)}
                     for k in range(slots)]

        def compute(k, it, sp):
            for j, M in enumerate(MS):
                ok(L.bl_linear_decode_grouped(slot_arrs[k][(M, replica_of(it, j, R))], count, api.BL_BF16, M, 1e-6,
                                              RDY, sp), "bl_linear_decode_grouped")

        run = E2E(dev, [x_all_host], [[x] for x in xa], [[y] for y in ya], [[y] for y in yah], compute, stream)
        n_e2e = max(3, min(K_, 300))
        spst_eager = run.run(n_e2e, world)
        reps_g = max(3, (K_ + R - 1) // R)
        spst = run.run_graph(R, reps_g, world)
        e2e = {"value": round(world * bytes_step / spst / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": x_all_host.numel() * 2, "d2h_bytes_per_step": y_all_host.numel() * 4,
               "steps": R * reps_g, "pipelining": f"{slots} buffer slots; one upload and one download per step, "
                                                  "on their own streams; the steps captured as one CUDA graph "
                                                  f"of {R} steps (copies included), replayed",
               "eager_value": round(world * bytes_step / spst_eager / 1e9, 2),
               "eager_note": "the same loop launched call by call from Python (host-bound)"}
        api.bl_check_device_error(stream)

    return {
        "value": round(value, 2), "ms_per_step": round(med / K_, 6), "steps": K_, "timing": spread(ms),
        "config": {"workload": WORKLOAD, "tokens_per_step": sum(MS), "projections": count,
                   "weight_bytes_per_m": wbytes, "activation_bytes_per_step": sum(2 * xbytes[M] for M in MS),
                   "weight_replicas": R,
                   "l2": f"{R} rotating packed-weight replicas ({R * wbytes / 2**20:.0f} MiB > 3x L2), "
                         "a different one for every launch",
                   "parallelism": f"replicas x{world}",
                   "launch": "each timed region = exactly --steps steps as one CUDA graph, 3 fused launches each"},
        "roofline": roof, "e2e": e2e, "alt_paths": alt, "gpu_launches": K_ * len(MS),
        "clocks": clk.summary(),
    }


def cpu_decode125m():
    import numpy as np
    import oracle
    wbytes, xbytes = step_bytes()
    items = []
    for _, W, X in workloads.decode125m(seed=1, M=max(MS)):
        packed, g, wq = oracle.quant_weights(W.numpy())
        items.append((wq, g, X.float().numpy().astype(np.float32)))
    t0 = time.perf_counter()
    for M in MS:
        for (wq, g, X) in items:
            xq, s = oracle.quant_act(X[:M])
            oracle.rescale(oracle.contract(xq, wq), g, s[:, None])
    secs = time.perf_counter() - t0
    bytes_step = sum(wbytes + 2 * xbytes[M] for M in MS)
    return {"value": round(bytes_step / secs / 1e9, 4), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "one whole step (84 projections at M = 1, 4, 8: act quant, int64 contraction, rescale); "
                      "OpenMP over token rows"}


# =============================================================================
# Config 1: one BitLinear 768 -> 2048, M = 16, fp32 W and X


def bench_single(args, world, local, dev, pk):
    from ternary_quantized_linear_bitlinear_b200 import api
    L = api.lib()
    W, X = workloads.single()
    N, K = W.shape
    M = X.shape[0]
    Wd, Xd = W.to(dev), X.to(dev)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    ws = torch.empty(api.linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    packed = torch.empty(N, K // 4, dtype=torch.uint8, device=dev)
    gamma = torch.empty(4, dtype=torch.float32, device=dev)
    wws = torch.empty(api.quant_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
    x_q = torch.empty(M, K, dtype=torch.int8, device=dev)
    s = torch.empty(M, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    CALLS = 64  # calls per timed region (one CUDA graph)
    F32 = api.BL_F32
    calls = {
        "bl_linear": lambda sp: ok(L.bl_linear(Wd.data_ptr(), F32, Xd.data_ptr(), F32, M, N, K, None, 1e-6,
                                               ws.data_ptr(), ws.numel(), Y.data_ptr(), sp), "bl_linear"),
        "bl_quant_weights": lambda sp: ok(L.bl_quant_weights(Wd.data_ptr(), F32, N, K, packed.data_ptr(),
                                                             gamma.data_ptr(), wws.data_ptr(), wws.numel(), sp),
                                          "bl_quant_weights"),
        "bl_quant_act": lambda sp: ok(L.bl_quant_act(Xd.data_ptr(), F32, M, K, None, 1e-6, x_q.data_ptr(),
                                                     s.data_ptr(), sp), "bl_quant_act"),
        "bl_forward": lambda sp: ok(L.bl_forward(packed.data_ptr(), gamma.data_ptr(), x_q.data_ptr(), s.data_ptr(),
                                                 M, N, K, Y.data_ptr(), None, sp), "bl_forward"),
    }
    # algorithmic bytes: inputs read once, outputs written once
    abytes = {"bl_linear": 4 * N * K + 4 * M * K + 4 * M * N,
              "bl_quant_weights": 4 * N * K + N * K // 4 + 4,
              "bl_quant_act": 4 * M * K + M * K + 4 * M,
              "bl_forward": N * K // 4 + M * K + 4 * M + 4 * M * N}
    res = {}
    with Clocks(local, "single") as clk:
        for name, fn in calls.items():
            def many(sp, fn=fn):
                for _ in range(CALLS):
                    fn(sp)
            g = graph_of(many, stream)
            ms = time_regions(g.replay, stream, world, min_ms=args.min_timed_ms / 4)
            us = statistics.median(ms) * 1e3 / CALLS
            res[name] = {"us_per_call": round(us, 3), "gbs": round(abytes[name] / (us * 1e-6) / 1e9, 1),
                         "algorithmic_bytes": abytes[name]}
            del g
    api.bl_check_device_error(stream)
    us = res["bl_linear"]["us_per_call"]
    out = {"config": {"workload": "single: BitLinear 768 -> 2048, M = 16; W fp32 ~N(0, 0.02^2); X fp32 ~N(0, 1) "
                                  "with 4 channels x20", "calls_per_region": CALLS,
                      "l2": "W (6.3 MB) stays in L2 between calls: a latency figure, not a bandwidth one"},
           "value": round(M / (us * 1e-6), 1), "unit": "tokens/s (whole bl_linear call)",
           "steps": res,
           "roofline": roofline_hbm("bl_linear: k_absmean_partial, k_ternary_pack, k_decode (fused act quant)",
                                    abytes["bl_linear"], us, pk,
                                    note="launch-latency bound: 6.3 MB of W per call, four launches"),
           "clocks": clk.summary()}
    if not args.no_e2e:
        slots = 2
        Wh, Xh = pinned(W), pinned(X)
        din = [[torch.empty_like(Wd), torch.empty_like(Xd)] for _ in range(slots)]
        dout = [[torch.empty_like(Y)] for _ in range(slots)]
        hout = [[torch.empty(M, N, dtype=torch.float32).pin_memory()] for _ in range(slots)]
        wss = [torch.empty_like(ws) for _ in range(slots)]

        def compute(k, it, sp):
            ok(L.bl_linear(din[k][0].data_ptr(), F32, din[k][1].data_ptr(), F32, M, N, K, None, 1e-6,
                           wss[k].data_ptr(), wss[k].numel(), dout[k][0].data_ptr(), sp), "bl_linear")

        spc = E2E(dev, [Wh, Xh], din, dout, hout, compute, stream).run(200, world)
        out["e2e"] = {"value": round(M / spc, 1), "unit": "tokens/s", "h2d_bytes_per_step": nbytes([Wh, Xh]),
                      "d2h_bytes_per_step": 4 * M * N, "steps": 200,
                      "pipelining": f"{slots} buffer slots, upload / compute / download streams"}
    if not args.no_cpu_baseline:
        import oracle
        Wn, Xn = W.numpy(), X.numpy()

        def one():
            t0 = time.perf_counter()
            oracle.linear(Wn, Xn)
            return time.perf_counter() - t0

        one()
        reps = 5
        t_all = statistics.median(one() for _ in range(reps))
        oracle.set_num_threads(1)
        t_one = statistics.median(one() for _ in range(reps))
        oracle.set_num_threads(oracle.num_threads())
        out["cpu_baseline"] = {"value": round(M / t_all, 1), "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle", "single_thread_value": round(M / t_one, 1),
                               "sample": f"the whole call (weight quant, act quant, int64 contraction, rescale), "
                                         f"median of {reps}; also on one thread"}
    return out


# =============================================================================
# Prefill-shaped layers (configs 3, 4 prefill, 5)


def layer_groups(names):
    """Projections sharing one input, as one grouped launch each: q,k,v | o |
    gate,up | down."""
    return [[names.index(n) for n in g] for g in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))]


class PrefillLayer:
    """One layer's projections on the device: pre-quantized engine inputs and
    per-call (bl_linear) inputs."""

    def __init__(self, dev, items, gains=None, share_x=False):
        from ternary_quantized_linear_bitlinear_b200 import api
        self.api = api
        self.L = api.lib()
        self.dev = dev
        self.names = [it[0] for it in items]
        self.groups = layer_groups(self.names)
        self.M = items[0][2].shape[0]
        self.rows = []
        gains = gains or [None] * len(items)
        for (name, W, X), g in zip(items, gains):
            Wd, Xd = W.to(dev), X.to(dev)
            gd = None if g is None else g.to(dev)
            packed, gamma = api.bl_quant_weights(Wd)
            x_q, s = api.bl_quant_act(Xd, gd, workloads.SUBLN_EPS)
            N, K = W.shape
            Y = torch.empty(self.M, N, dtype=torch.float32, device=dev)
            self.rows.append(dict(name=name, W=Wd, X=Xd, gain=gd, packed=packed, gamma=gamma, x_q=x_q, s=s, Y=Y,
                                  N=N, K=K, wdt=api._DTYPES[W.dtype], xdt=api._DTYPES[X.dtype]))
        self.ws = torch.empty(max(api.linear_workspace_bytes(self.M, r["N"], r["K"]) for r in self.rows),
                              dtype=torch.uint8, device=dev)
        self.ops = sum(2 * self.M * r["N"] * r["K"] for r in self.rows)
        self.garrs = []
        for g in self.groups:
            arr = (api.Problem * len(g))()
            r0 = self.rows[g[0]]
            for j, i in enumerate(g):
                r = self.rows[i]
                # projections of a group share the first member's activation, as in a layer
                arr[j] = api.Problem(r["packed"].data_ptr(), r["gamma"].data_ptr(), r0["x_q"].data_ptr(),
                                     r0["s"].data_ptr(), r["Y"].data_ptr(), None, r["N"], r["K"])
            self.garrs.append((arr, len(g)))

    def engine(self, sp):
        for r in self.rows:
            ok(self.L.bl_forward(r["packed"].data_ptr(), r["gamma"].data_ptr(), r["x_q"].data_ptr(),
                                 r["s"].data_ptr(), self.M, r["N"], r["K"], r["Y"].data_ptr(), None, sp), "bl_forward")

    def engine_grouped(self, sp):
        for arr, n in self.garrs:
            ok(self.L.bl_forward_grouped(arr, n, self.M, 0, sp), "bl_forward_grouped")

    def per_call_grouped(self, sp):
        """The per-call path as a layer runs it: per group of projections
        sharing an input (q,k,v | o | gate,up | down) one bl_linear_grouped
        call: grouped weight quantization, one act quant, one grouped GEMM."""
        api = self.api
        if not hasattr(self, "_lg"):
            self._lg = []
            need = 0
            for g in self.groups:
                arr = (api.LinearProblem * len(g))()
                for j, i in enumerate(g):
                    r = self.rows[i]
                    arr[j] = api.LinearProblem(r["W"].data_ptr(), r["Y"].data_ptr(), r["N"])
                r0 = self.rows[g[0]]
                need = max(need, int(self.L.bl_linear_grouped_workspace_bytes(arr, len(g), self.M, r0["K"])))
                self._lg.append((arr, len(g), r0))
            self._lg_ws = torch.empty(need, dtype=torch.uint8, device=self.dev)
        for arr, n, r0 in self._lg:
            ok(self.L.bl_linear_grouped(arr, n, r0["wdt"], r0["X"].data_ptr(), r0["xdt"], self.M, r0["K"],
                                        None if r0["gain"] is None else r0["gain"].data_ptr(), workloads.SUBLN_EPS,
                                        self._lg_ws.data_ptr(), self._lg_ws.numel(), sp), "bl_linear_grouped")

    def per_call_layer(self, sp):
        """The per-call path with the layer's weights quantized together: one
        bl_quant_weights_grouped over all projections (at most eight), then
        per group of projections sharing an input one act quant and one
        grouped GEMM."""
        api = self.api
        if not hasattr(self, "_pl"):
            n = len(self.rows)
            warr = (api.WeightProblem * n)()
            for i, r in enumerate(self.rows):
                warr[i] = api.WeightProblem(r["W"].data_ptr(), r["N"], r["K"], r["packed"].data_ptr(),
                                            r["gamma"].data_ptr())
            wsz = int(self.L.bl_quant_weights_workspace_bytes(self.rows[0]["N"], self.rows[0]["K"]))
            self._pl = (warr, n, torch.empty(wsz, dtype=torch.uint8, device=self.dev))
        warr, n, wws = self._pl
        ok(self.L.bl_quant_weights_grouped(warr, n, self.rows[0]["wdt"], wws.data_ptr(), wws.numel(), sp),
           "bl_quant_weights_grouped")
        for g, (arr, ng) in zip(self.groups, self.garrs):
            r0 = self.rows[g[0]]
            ok(self.L.bl_quant_act(r0["X"].data_ptr(), r0["xdt"], self.M, r0["K"],
                                   None if r0["gain"] is None else r0["gain"].data_ptr(), workloads.SUBLN_EPS,
                                   r0["x_q"].data_ptr(), r0["s"].data_ptr(), sp), "bl_quant_act")
            ok(self.L.bl_forward_grouped(arr, ng, self.M, 0, sp), "bl_forward_grouped")

    def per_call(self, sp, rows=None, Ws=None, Xs=None, Ys=None):
        for i, r in enumerate(self.rows):
            W = r["W"] if Ws is None else Ws[i]
            X = r["X"] if Xs is None else Xs[i]
            Y = r["Y"] if Ys is None else Ys[i]
            ok(self.L.bl_linear(W.data_ptr(), r["wdt"], X.data_ptr(), r["xdt"], self.M, r["N"], r["K"],
                                None if r["gain"] is None else r["gain"].data_ptr(), workloads.SUBLN_EPS,
                                self.ws.data_ptr(), self.ws.numel(), Y.data_ptr(), sp), "bl_linear")


def time_layer_fns(layer, fns, stream, world, args, reps_per_region=1):
    out = {}
    for label, fn in fns.items():
        def many(sp, fn=fn):
            for _ in range(reps_per_region):
                fn(sp)
        g = graph_of(many, stream)
        ms = time_regions(g.replay, stream, world, min_reps=20, min_ms=args.min_timed_ms / len(fns))
        per = statistics.median(ms) / reps_per_region
        out[label] = {"ms_per_layer": round(per, 4), "tops": round(layer.ops / (per * 1e-3) / 1e12, 1),
                      "timing": spread(ms)}
        del g
    return out


def e2e_per_call(layer, dev, stream, world, steps, slots=1):
    """The per-call path with every input (W, X) uploaded and every Y
    downloaded each step."""
    host_in = []
    for r in layer.rows:
        host_in += [pinned(r["W"].cpu()), pinned(r["X"].cpu())]
    din = [[torch.empty_like(h, device=dev) for h in host_in] for _ in range(slots)]
    dout = [[torch.empty_like(r["Y"]) for r in layer.rows] for _ in range(slots)]
    hout = [[torch.empty(r["Y"].shape, dtype=torch.float32).pin_memory() for r in layer.rows] for _ in range(slots)]

    def compute(k, it, sp):
        layer.per_call(sp, Ws=din[k][0::2], Xs=din[k][1::2], Ys=dout[k])

    spst = E2E(dev, host_in, din, dout, hout, compute, stream).run(steps, world, warm=1)
    return spst, nbytes(host_in), sum(4 * r["Y"].numel() for r in layer.rows)


def cpu_layer(items, tokens, gains=None, quant_weights=True):
    """Oracle on a bounded sample: the first `tokens` rows of every
    projection (weight quant when asked, act quant, int64 contraction,
    rescale).  Returns (seconds, ops of the sample)."""
    import oracle
    gains = gains or [None] * len(items)
    prepped = []
    for (name, W, X), g in zip(items, gains):
        prepped.append((W.float().numpy(), X[:tokens].float().numpy(), None if g is None else g.numpy()))
    wq_cache = []
    if not quant_weights:
        wq_cache = [oracle.quant_weights(W)[1:] for W, _, _ in prepped]
    ops = 0
    t0 = time.perf_counter()
    for i, (W, X, g) in enumerate(prepped):
        gamma, wq = oracle.quant_weights(W)[1:] if quant_weights else wq_cache[i]
        xq, s = oracle.quant_act(X, g, workloads.SUBLN_EPS)
        oracle.rescale(oracle.contract(xq, wq), gamma, s[:, None])
        ops += 2 * X.shape[0] * W.shape[0] * W.shape[1]
    return time.perf_counter() - t0, ops


def bench_prefill1b4(args, world, local, dev, pk):
    from ternary_quantized_linear_bitlinear_b200 import api
    items = workloads.prefill1b4()
    layer = PrefillLayer(dev, items)
    stream = torch.cuda.Stream(device=dev)
    with Clocks(local, "prefill1b4") as clk:
        res = time_layer_fns(layer, {"engine": layer.engine, "engine_grouped": layer.engine_grouped,
                                     "per_call": layer.per_call, "per_call_grouped": layer.per_call_grouped,
                                     "per_call_layer": layer.per_call_layer},
                             stream, world, args)
        # FFN activation + SubLN + act quant feeding the down projection (bl_ffn_act_quant)
        M, F = layer.M, workloads.PREFILL1B4["ffn"]
        gate = workloads.normal((M, F), 1.5, 60).to(dev)
        up = workloads.normal((M, F), 1.0, 61).to(dev)
        fgain = workloads.uniform((F,), 0.9, 1.1, 62).to(dev)
        fxq = torch.empty(M, F, dtype=torch.int8, device=dev)
        fs = torch.empty(M, dtype=torch.float32, device=dev)
        L = api.lib()
        g = graph_of(lambda sp: ok(L.bl_ffn_act_quant(gate.data_ptr(), up.data_ptr(), M, F, fgain.data_ptr(), 1e-6,
                                                      fxq.data_ptr(), fs.data_ptr(), sp), "bl_ffn_act_quant"), stream)
        ffn_us = statistics.median(time_regions(g.replay, stream, world, min_ms=50)) * 1e3
        del g
        # the FFN block from x_q to the down projection's input, two ways:
        # (a) gate, up in one grouped GEMM writing both Y, then bl_ffn_act_quant
        # (b) bl_forward_glu (only h written), then bl_quant_act(h) with SubLN
        ig, iu = layer.names.index("gate"), layer.names.index("up")
        rg, ru = layer.rows[ig], layer.rows[iu]
        gu = (api.Problem * 2)()
        for j, r in enumerate((rg, ru)):
            gu[j] = api.Problem(r["packed"].data_ptr(), r["gamma"].data_ptr(), rg["x_q"].data_ptr(), rg["s"].data_ptr(),
                                r["Y"].data_ptr(), None, r["N"], r["K"])
        hbuf = torch.empty(M, F, dtype=torch.float32, device=dev)

        def ffn_sep(sp):
            ok(L.bl_forward_grouped(gu, 2, M, 0, sp), "bl_forward_grouped")
            ok(L.bl_ffn_act_quant(rg["Y"].data_ptr(), ru["Y"].data_ptr(), M, F, fgain.data_ptr(), 1e-6,
                                  fxq.data_ptr(), fs.data_ptr(), sp), "bl_ffn_act_quant")

        def ffn_glu(sp):
            ok(L.bl_forward_glu(rg["packed"].data_ptr(), rg["gamma"].data_ptr(), ru["packed"].data_ptr(),
                                ru["gamma"].data_ptr(), rg["x_q"].data_ptr(), rg["s"].data_ptr(), M, F, rg["K"],
                                hbuf.data_ptr(), sp), "bl_forward_glu")
            ok(L.bl_quant_act(hbuf.data_ptr(), api.BL_F32, M, F, fgain.data_ptr(), 1e-6, fxq.data_ptr(),
                              fs.data_ptr(), sp), "bl_quant_act")

        ffn_block = {}
        for label, fn in (("gate_up_then_ffn_act_quant", ffn_sep), ("glu_then_quant_act", ffn_glu)):
            g = graph_of(fn, stream)
            us = statistics.median(time_regions(g.replay, stream, world, min_ms=50)) * 1e3
            ffn_block[label] = {"us": round(us, 2)}
            del g
    api.bl_check_device_error(stream)
    ffn_bytes = 2 * M * F * 4 + M * F + 4 * M
    best = "engine_grouped" if res["engine_grouped"]["tops"] >= res["engine"]["tops"] else "engine"
    out = {"config": {"workload": "prefill1b4: hidden 1536, FFN 4096, q,o 1536^2, k,v 512x1536, gate,up 4096x1536, "
                                  "down 1536x4096, M = 8192; W bf16 ~N(0, 0.02^2), X bf16 = 0.5 t(3)",
                      "ops_per_layer": layer.ops,
                      "l2": "inputs and outputs of the layer total > 700 MB"},
           "value": max(res[k]["tops"] for k in PER_CALL),
           "unit": "TOPS (per-call path: weights quantized in the call)",
           **res,
           "engine_grouped_launches": "q,k,v | o | gate,up | down (shared-input projections in one launch)",
           "roofline": roofline_tensor("k_prefill_tc", layer.ops, res[best]["ms_per_layer"], pk, best),
           "per_call_frac": round(max(res[k]["tops"] for k in PER_CALL) / pk["int8"], 4),
           "per_call_paths": "per_call: bl_linear x7; per_call_grouped: bl_linear_grouped per group of "
                             "projections sharing an input; per_call_layer: one bl_quant_weights_grouped over "
                             "the layer's 7 matrices, then per group bl_quant_act + bl_forward_grouped",
           "ffn_act_quant": {"shape": f"gate, up [{M}, {F}] f32 -> x_q [{M}, {F}] (ReLU^2 gate, SubLN)",
                             "us": round(ffn_us, 2), "gbs": round(ffn_bytes / (ffn_us * 1e-6) / 1e9, 1),
                             "frac_hbm": round(ffn_bytes / (ffn_us * 1e-6) / 1e9 / pk["hbm"], 4)},
           "ffn_block": {**ffn_block, "from": "x_q of the FFN input", "to": "x_q, s of the down projection",
                         "y_bytes_written": {"gate_up_then_ffn_act_quant": 2 * 4 * M * F,
                                             "glu_then_quant_act": 4 * M * F}},
           "clocks": clk.summary()}
    if not args.no_e2e:
        spst, hin, hout = e2e_per_call(layer, dev, stream, world, steps=4)
        out["e2e"] = {"value": round(layer.ops / spst / 1e12, 2), "unit": "TOPS", "h2d_bytes_per_step": hin,
                      "d2h_bytes_per_step": hout, "steps": 4,
                      "path": "per-call bl_linear x7 with W and X uploaded and Y downloaded every step"}
    if not args.no_cpu_baseline:
        import oracle
        secs, ops = cpu_layer(items, 32)
        out["cpu_baseline"] = {"value": round(ops / secs / 1e12, 6), "unit": "TOPS", "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": "per-call path on the first 32 of 8192 tokens of every projection "
                                         "(weight quant, act quant, int64 contraction, rescale)"}
    return out


def bench_layer3b(args, world, local, dev, pk):
    from ternary_quantized_linear_bitlinear_b200 import api
    L = api.lib()
    stream = torch.cuda.Stream(device=dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    out = {"config": {"workload": "layer3b: hidden 3200, FFN 8640, q,k,v,o 3200^2, gate,up 8640x3200, "
                                  "down 3200x8640; W fp32 ~N(0, 0.015^2) absmean-quantized once; X bf16 ~N(0, 1) "
                                  "with 1 % of channels x30; decode M = 1, prefill M = 2048"}}
    # ---- decode, M = 1: all seven projections in one fused grouped launch --
    items1 = workloads.layer3b(M=1)
    packed, gammas = [], []
    for _, W, _ in items1:
        p, g = api.bl_quant_weights(W.to(dev))
        packed.append(p)
        gammas.append(g)
    flat = torch.cat([p.view(-1) for p in packed])
    wbytes = flat.numel()
    offs, o = [], 0
    for p in packed:
        offs.append(o)
        o += p.numel()
    R = max(2, (3 * l2) // wbytes + 1)
    reps = [flat] + [flat.clone() for _ in range(R - 1)]
    xs = [X.to(dev) for _, _, X in items1]
    xbytes = sum(2 * X.numel() for X in xs)
    Ys = [torch.empty(1, W.shape[0], dtype=torch.float32, device=dev) for _, W, _ in items1]

    def arr_of(rep, sel, xbuf=None, ybuf=None):
        xbuf = xs if xbuf is None else xbuf
        ybuf = Ys if ybuf is None else ybuf
        a = (api.DecodeProblem * len(sel))()
        for j, i in enumerate(sel):
            N, K = items1[i][1].shape
            a[j] = api.DecodeProblem(reps[rep].data_ptr() + offs[i], gammas[i].data_ptr(), xbuf[i].data_ptr(), None,
                                     ybuf[i].data_ptr(), None, None, None, N, K)
        return a

    allsel = list(range(len(items1)))
    arrs = [arr_of(r, allsel) for r in range(R)]
    RDY = api.BL_FWD_WEIGHTS_READY
    nl = 4 * R

    def dec(sp):
        for i in range(nl):
            ok(L.bl_linear_decode_grouped(arrs[i % R], len(allsel), api.BL_BF16, 1, 1e-6, RDY, sp),
               "bl_linear_decode_grouped")

    names = [n for n, _, _ in items1]
    stages = layer_groups(names)
    st_arrs = [[arr_of(r, sel) for sel in stages] for r in range(R)]

    def dep(sp):
        for i in range(nl):
            for a, sel in zip(st_arrs[i % R], stages):
                ok(L.bl_linear_decode_grouped(a, len(sel), api.BL_BF16, 1, 1e-6, RDY, sp), "bl_linear_decode_grouped")

    with Clocks(local, "layer3b_decode") as clk:
        g = graph_of(dec, stream)
        ms = time_regions(g.replay, stream, world, min_ms=args.min_timed_ms / 2)
        us = statistics.median(ms) * 1e3 / nl
        del g
        g = graph_of(dep, stream)
        us_dep = statistics.median(time_regions(g.replay, stream, world, min_ms=50)) * 1e3 / nl
        del g
    api.bl_check_device_error(stream)
    out["decode_m1"] = {
        "us_per_layer": round(us, 3), "gbs": round((wbytes + xbytes) / (us * 1e-6) / 1e9, 1), "timing": spread(ms),
        "weight_replicas": R, "launch": "one fused grouped launch over the 7 projections, its own replica each",
        "roofline": roofline_hbm("k_decode (fused act quant + GEMV, 7 problems)", wbytes + xbytes, us, pk),
        "dependent_4_launches_us_per_layer": round(us_dep, 3),
        "dependent_note": "qkv | o | gate,up | down as four ordered launches (the attention itself is out of scope)",
        "clocks": clk.summary()}
    out["value"] = out["decode_m1"]["gbs"]
    out["unit"] = "GB/s (decode M = 1)"
    if not args.no_e2e:
        slots = 2
        xh = [pinned(X.cpu()) for X in xs]
        din = [[torch.empty_like(x) for x in xs] for _ in range(slots)]
        dout = [[torch.empty_like(y) for y in Ys] for _ in range(slots)]
        hout = [[torch.empty(y.shape, dtype=torch.float32).pin_memory() for y in Ys] for _ in range(slots)]
        sarr = [[arr_of(r, allsel, din[k], dout[k]) for r in range(R)] for k in range(slots)]

        def compute(k, it, sp):
            ok(L.bl_linear_decode_grouped(sarr[k][it % R], len(allsel), api.BL_BF16, 1, 1e-6, RDY, sp),
               "bl_linear_decode_grouped")

        run = E2E(dev, xh, din, dout, hout, compute, stream)
        spst_eager = run.run(100, world)
        spst = run.run_graph(2 * R, 10, world)
        out["decode_m1"]["e2e"] = {"value": round((wbytes + xbytes) / spst / 1e9, 1), "unit": "GB/s",
                                   "h2d_bytes_per_step": nbytes(xh), "d2h_bytes_per_step": nbytes(Ys),
                                   "steps": 20 * R, "pipelining": f"2 buffer slots; {2 * R} steps per CUDA graph "
                                                                 "(copies included), replayed",
                                   "eager_value": round((wbytes + xbytes) / spst_eager / 1e9, 1)}
    if not args.no_cpu_baseline:
        import oracle
        secs, _ = cpu_layer(items1, 1, quant_weights=False)
        out["decode_m1"]["cpu_baseline"] = {"value": round((wbytes + xbytes) / secs / 1e9, 4), "unit": "GB/s",
                                            "cores": oracle.num_threads(), "kind": "oracle",
                                            "sample": "the whole layer at M = 1 (act quant, int64 contraction, "
                                                      "rescale; weights quantized beforehand)"}
    del reps, arrs, st_arrs
    # ---- prefill, M = 2048 --------------------------------------------------
    items = workloads.layer3b(M=2048)
    layer = PrefillLayer(dev, items)
    with Clocks(local, "layer3b_prefill") as clk:
        res = time_layer_fns(layer, {"engine": layer.engine, "engine_grouped": layer.engine_grouped}, stream,
                             world, args)
    api.bl_check_device_error(stream)
    best = "engine_grouped" if res["engine_grouped"]["tops"] >= res["engine"]["tops"] else "engine"
    out["prefill_m2048"] = {**res, "ops_per_layer": layer.ops,
                            "roofline": roofline_tensor("k_prefill_tc", layer.ops, res[best]["ms_per_layer"], pk,
                                                        best),
                            "clocks": clk.summary()}
    if not args.no_e2e:
        # engine path with x_q uploaded and Y downloaded per step
        slots = 2
        xh = [pinned(r["x_q"].cpu()) for r in layer.rows] + [pinned(r["s"].cpu()) for r in layer.rows]
        din = [[torch.empty_like(h, device=dev) for h in xh] for _ in range(slots)]
        dout = [[torch.empty_like(r["Y"]) for r in layer.rows] for _ in range(slots)]
        hout = [[torch.empty(r["Y"].shape, dtype=torch.float32).pin_memory() for r in layer.rows]
                for _ in range(slots)]
        n = len(layer.rows)

        def compute(k, it, sp):
            for i, r in enumerate(layer.rows):
                ok(L.bl_forward(r["packed"].data_ptr(), r["gamma"].data_ptr(), din[k][i].data_ptr(),
                                din[k][n + i].data_ptr(), layer.M, r["N"], r["K"], dout[k][i].data_ptr(), None, sp),
                   "bl_forward")

        spst = E2E(dev, xh, din, dout, hout, compute, stream).run(10, world, warm=1)
        out["prefill_m2048"]["e2e"] = {"value": round(layer.ops / spst / 1e12, 2), "unit": "TOPS",
                                       "h2d_bytes_per_step": nbytes(xh),
                                       "d2h_bytes_per_step": sum(4 * r["Y"].numel() for r in layer.rows),
                                       "steps": 10, "path": "bl_forward x7, x_q and s uploaded, Y downloaded"}
    if not args.no_cpu_baseline:
        import oracle
        secs, ops = cpu_layer(items, 16, quant_weights=False)
        out["prefill_m2048"]["cpu_baseline"] = {"value": round(ops / secs / 1e12, 6), "unit": "TOPS",
                                                "cores": oracle.num_threads(), "kind": "oracle",
                                                "sample": "first 16 of 2048 tokens of every projection"}
    return out


def bench_qat4b(args, world, local, dev, pk):
    from ternary_quantized_linear_bitlinear_b200 import api
    items4 = workloads.qat4b()
    items = [(n, W, X) for n, W, X, _ in items4]
    gains = [g for _, _, _, g in items4]
    layer = PrefillLayer(dev, items, gains)
    stream = torch.cuda.Stream(device=dev)
    with Clocks(local, "qat4b") as clk:
        res = time_layer_fns(layer, {"per_call": layer.per_call, "per_call_grouped": layer.per_call_grouped,
                                     "per_call_layer": layer.per_call_layer,
                                     "engine_grouped": layer.engine_grouped}, stream, world, args)
    api.bl_check_device_error(stream)
    out = {"config": {"workload": "qat4b: hidden 2560, FFN 9728, q,k,v,o 2560^2, gate,up 9728x2560, down 2560x9728, "
                                  "M = 16 x 2048 = 32768; bf16 master W ~N(0, 0.02^2) re-quantized every call; SubLN "
                                  "(gain ~U(0.9, 1.1), eps 1e-6) fused into the act quant before o_proj and "
                                  "down_proj", "ops_per_layer": layer.ops},
           "value": max(res[k]["tops"] for k in PER_CALL), "unit": "TOPS (per-call path)",
           **res,
           "roofline": roofline_tensor("k_prefill_tc", layer.ops, min(res[k]["ms_per_layer"] for k in PER_CALL), pk,
                                       max(PER_CALL, key=lambda k: res[k]["tops"])),
           "engine_frac": round(res["engine_grouped"]["tops"] / pk["int8"], 4),
           "clocks": clk.summary()}
    if not args.no_e2e:
        spst, hin, hout = e2e_per_call(layer, dev, stream, world, steps=3)
        out["e2e"] = {"value": round(layer.ops / spst / 1e12, 2), "unit": "TOPS", "h2d_bytes_per_step": hin,
                      "d2h_bytes_per_step": hout, "steps": 3,
                      "path": "per-call bl_linear x7 with W and X uploaded and Y downloaded every step"}
    if not args.no_cpu_baseline:
        import oracle
        secs, ops = cpu_layer(items, 8, gains)
        out["cpu_baseline"] = {"value": round(ops / secs / 1e12, 6), "unit": "TOPS", "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": "per-call path on the first 8 of 32768 tokens of every projection "
                                         "(weight quant, SubLN act quant, int64 contraction, rescale)"}
    return out


# =============================================================================
# Reference arm: the CPU oracle on the headline workload


def reference(args, rank, world):
    """The CPU oracle as the reference arm, on the same metric and workload;
    each step is one projection (cycling through the 84 and M = 1, 4, 8),
    rows of W subsampled so the run stays within a few minutes."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    items = []
    for _, W, X in workloads.decode125m(seed=1, M=max(MS)):
        packed, g, wq = oracle.quant_weights(W.numpy())
        items.append((wq, g, X.float().numpy().astype(np.float32)))
    jobs = [(M, i) for M in MS for i in range(len(items))]
    total_steps = args.steps + max(3, args.warmup)
    budget_s = args.ref_budget_s / max(1, total_steps)
    # calibrate the oracle's rows-per-second on one projection (not timed)
    wq, g, X = items[4]
    t0 = time.perf_counter()
    xq, s = oracle.quant_act(X[:8])
    oracle.rescale(oracle.contract(xq, wq[:256]), g, s[:, None])
    per_row = (time.perf_counter() - t0) / 256
    rows = int(max(16, min(4096, budget_s / max(per_row, 1e-9))))
    done_bytes = 0
    t_start = None
    for it in range(total_steps):
        if it == max(3, args.warmup):
            t_start = time.perf_counter()
            done_bytes = 0
        M, i = jobs[it % len(jobs)]
        wq, g, X = items[i]
        n = min(rows, wq.shape[0])
        xq, s = oracle.quant_act(X[:M])
        oracle.rescale(oracle.contract(xq, wq[:n]), g, s[:, None])
        done_bytes += n * wq.shape[1] // 4 + 2 * M * wq.shape[1]
    secs = time.perf_counter() - t_start
    value = done_bytes / secs / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(secs * 1e3 / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic", "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"per step one projection (cycling 84 x M in 1,4,8), first {rows} rows of W"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def native(args, rank, world, local):
    dev = torch.device("cuda", torch.cuda.current_device())
    pk = peaks()
    only = [c.strip() for c in args.only.split(",") if c.strip()]
    if "decode125m" not in only:
        # a run of other workloads alone (e.g. under a profiler): no headline
        out = {"metric": METRIC, "note": "headline workload (decode125m) not requested"}
        if rank == 0:
            out["configs"] = {name: fn(args, 1, local, dev, pk)
                              for name, fn in (("single", bench_single), ("prefill1b4", bench_prefill1b4),
                                               ("layer3b", bench_layer3b), ("qat4b", bench_qat4b)) if name in only}
        return out
    head = bench_decode125m(args, rank, world, local, dev, pk)
    out = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": head["steps"],
        "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": head["config"], "roofline": head["roofline"], "e2e": head["e2e"], "alt_paths": head["alt_paths"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "timing": head["timing"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_decode125m()
    configs = {}
    # the other workloads run on rank 0 only (one GPU's worth; the headline is
    # the weak-scaling measurement)
    if rank == 0:
        for name, fn in (("single", bench_single), ("prefill1b4", bench_prefill1b4), ("layer3b", bench_layer3b),
                         ("qat4b", bench_qat4b)):
            if name in only:
                configs[name] = fn(args, 1, local, dev, pk)
                torch.cuda.empty_cache()
    if configs:
        out["configs"] = configs
    return out


def main():
    args = parse()
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            out = reference(args, rank, world)
        else:
            out = native(args, rank, world, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
