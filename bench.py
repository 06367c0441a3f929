"""Benchmark: BitLinear decode over the 125M-shape decode workload.

One step = the decode hot path for every projection of all 12 layers
(q,o 768x768; k,v 256x768; gate,up 2048x768; down 768x2048 -- 84 problems)
at M = 1, 4 and 8 tokens: per M, ONE grouped launch that quantizes the bf16
activations, runs the ternary GEMV and rescales (bl_linear_decode_grouped).
The ternary weights (29/42/29 split) are packed once at load time.  Weight
bytes per step would fit in L2, so the packed weights are replicated and
every launch reads a different replica than the launches around it (the
replicas total more than 3x the L2 size).

Metric: decode GB/s = (packed weight bytes + bf16 activation bytes) per step
/ time, whole job, N GPUs = N independent replicas of the workload (weak
scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
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


def replica_of(step: int, j: int, replicas: int) -> int:
    """Weight replica read by launch j (the j-th M) of a step: consecutive
    launches never share weights (the launches of one step included), so no
    launch is fed from L2; a replica comes back every `replicas` launches."""
    return (len(MS) * step + j) % replicas


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="reference arm: seconds of oracle work over the whole run")
    ap.add_argument("--mode", default="all", choices=["all", "decode", "prefill"],
                    help="decode: the headline decode workload only; prefill: only the prefill measurement")
    return ap.parse_args()


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


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -- workload ----------------------------------------------------------------

def step_bytes():
    """Algorithmic bytes of one step: packed weights + x_q, per M."""
    shapes = workloads.decode125m_layer_shapes()
    L = workloads.DECODE125M["layers"]
    wbytes = L * sum(N * K // 4 for _, N, K, _ in shapes)
    xbytes = {M: L * sum(M * K for _, N, K, _ in shapes) for M in MS}
    return wbytes, xbytes


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
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
        self.path = os.path.join(os.environ.get("BL_CLOCKS_DIR") or tempfile.gettempdir(), f"clocks_rank{index}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
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
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


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


def native(args, rank, world, local):
    from ternary_quantized_linear_bitlinear_b200 import api

    dev = torch.device("cuda", torch.cuda.current_device())
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
    offs = []
    o = 0
    for p in packed0:
        offs.append(o)
        o += p.numel()
    replicas = [flat0] + [flat0.clone() for _ in range(R - 1)]

    # activations: one contiguous bf16 buffer per M (inputs of all 84 problems)
    # (per M, views into ONE input buffer and ONE output buffer for the whole
    # step, so the end-to-end run moves each step's data in one copy per way)
    xin, xq, sc, Y = {}, {}, {}, {}
    xin_host, y_host = {}, {}
    xlen = {M: sum(M * K for _, K in shapes) for M in MS}                  # multiples of 64: 128-byte aligned views
    ylen = {M: sum(M * N for N, _ in shapes) + 4 * len(items) for M in MS}  # per-problem slots padded to 4
    x_all_host = torch.cat([torch.cat([X[:M].contiguous().view(-1) for _, _, X in items]) for M in MS]).pin_memory()
    x_all = x_all_host.to(dev)
    y_all = torch.empty(sum(ylen.values()), dtype=torch.float32, device=dev)
    y_all_host = torch.empty_like(y_all, device="cpu").pin_memory()
    xo = yo = 0
    for M in MS:
        xin_host[M], xin[M] = x_all_host[xo:xo + xlen[M]], x_all[xo:xo + xlen[M]]
        Y[M], y_host[M] = y_all[yo:yo + ylen[M]], y_all_host[yo:yo + ylen[M]]
        xo += xlen[M]
        yo += ylen[M]
        xq[M] = torch.empty(xin[M].numel(), dtype=torch.int8, device=dev)  # two-launch path only
        sc[M] = torch.empty(len(items) * SPAD[M], dtype=torch.float32, device=dev)

    def views(M, xbuf=None, ybuf=None):
        """Per-problem device views into the contiguous buffers (16-byte aligned)."""
        xbuf = xin if xbuf is None else xbuf
        ybuf = Y if ybuf is None else ybuf
        out = []
        xo = yo = 0
        for i, (N, K) in enumerate(shapes):
            out.append((xbuf[M][xo:xo + M * K], xq[M][xo:xo + M * K], sc[M][i * SPAD[M]:i * SPAD[M] + M],
                        ybuf[M][yo:yo + M * N], N, K))
            xo += M * K
            yo += (M * N + 3) // 4 * 4
        return out

    def fused_problems(M, rep, sel=None, xbuf=None, ybuf=None):
        v = views(M, xbuf, ybuf)
        idx = range(len(v)) if sel is None else sel
        arr = (api.DecodeProblem * len(idx))()
        base = replicas[rep].data_ptr()
        for j, i in enumerate(idx):
            X, _, _, y, N, K = v[i]
            arr[j] = api.DecodeProblem(base + offs[i], gammas[i].data_ptr(), X.data_ptr(), None, y.data_ptr(), None,
                                       None, None, N, K)
        return arr

    def two_launch_problems(M, rep):
        v = views(M)
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

    def replica(step, j):
        return replica_of(step, j, R)

    def launch_step(stream_ptr, rep):
        """One step: per M, ONE fused launch (act quant + GEMV + rescale, 84 problems)."""
        for j, M in enumerate(MS):
            rc = L.bl_linear_decode_grouped(fused[(M, replica(rep, j))], count, api.BL_BF16, M, 1e-6, RDY, stream_ptr)
            if rc:
                raise api.BitLinearError(rc, "bl_linear_decode_grouped")

    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream

    def graph_of(fn, reps):
        with torch.cuda.stream(stream):  # eager warm-up: also runs the one-time device set-up
            for r in range(reps):
                fn(sp, r)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                fn(stream.cuda_stream, r)
        torch.cuda.synchronize()
        return g

    def time_graph(g, replays):
        with torch.cuda.stream(stream):
            g.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(replays):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    # ---- capture one cycle (R steps, one per replica) as a CUDA graph ------
    g_step = graph_of(launch_step, R)

    K_, Wm = args.steps, max(3, args.warmup)
    cycles = max(1, (K_ + R - 1) // R)
    steps_timed = cycles * R
    for _ in range(max(1, (Wm + R - 1) // R)):
        g_step.replay()
    torch.cuda.synchronize()

    # ---- timed region: whole steps ----------------------------------------
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(cycles):
                g_step.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    ms_per_step = ms_total / steps_timed
    bytes_step = sum(wbytes + 2 * xbytes[M] for M in MS)  # packed W + bf16 X read by the fused kernel
    value = world * bytes_step * steps_timed / (ms_total * 1e-3) / 1e9
    api.bl_check_device_error(stream)

    # ---- the dominant kernel: every launch of the step is the fused GEMV ---
    dec_us = ev0.elapsed_time(ev1) * 1e3 / (steps_timed * len(MS))  # this rank's launches
    dec_bytes = bytes_step / len(MS)  # per launch, averaged over M
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    peak = float(peaks.get("hbm_gbs", 6650.0))
    achieved = dec_bytes / (dec_us * 1e-6) / 1e9
    roofline = {"bound": "hbm", "kernel": "k_decode<1, bf16> (fused act quant + ternary GEMV + rescale, 84 problems)",
                "achieved": round(achieved, 1), "peak": peak,
                "peak_source": "measured" if "hbm_gbs" in peaks else "fallback",
                "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": decode_traffic(),
                "avg_launch_us": round(dec_us, 3), "algorithmic_bytes_per_launch": int(dec_bytes)}

    # ---- secondary: the same step as two launches per M (act quant, GEMV) -
    alt = {}
    if not args.no_e2e:
        tl = {(M, r): two_launch_problems(M, r) for M in MS for r in range(R)}

        def two_step(stream_ptr, rep):
            for j, M in enumerate(MS):
                acts, fwd = tl[(M, replica(rep, j))]
                if L.bl_quant_act_grouped(acts, count, api.BL_BF16, M, 1e-6, stream_ptr):
                    raise RuntimeError("bl_quant_act_grouped")
                if L.bl_forward_grouped(fwd, count, M, RDY, stream_ptr):
                    raise RuntimeError("bl_forward_grouped")

        g2 = graph_of(two_step, R)
        alt["two_launch_us_per_step"] = round(time_graph(g2, max(1, cycles // 4)) * 1e3 / (R * max(1, cycles // 4)), 3)
        del g2
        # layer order at M = 1: per layer qkv | o | gate, up | down (4 grouped launches, 48 per step)
        stages = []
        per_layer = len(workloads.decode125m_layer_shapes())
        for layer in range(count // per_layer):
            b0 = layer * per_layer
            for sel in ((0, 1, 2), (3,), (4, 5), (6,)):
                stages.append([b0 + j for j in sel])
        lay = {r: [fused_problems(1, r, sel) for sel in stages] for r in range(R)}

        def layered_step(stream_ptr, rep):
            for arr, sel in zip(lay[rep], stages):
                if L.bl_linear_decode_grouped(arr, len(sel), api.BL_BF16, 1, 1e-6, RDY, stream_ptr):
                    raise RuntimeError("bl_linear_decode_grouped")

        g3 = graph_of(layered_step, R)
        reps3 = max(1, cycles // 4)
        us3 = time_graph(g3, reps3) * 1e3 / (R * reps3)
        alt["layered_m1_us_per_step"] = round(us3, 3)
        alt["layered_m1_gbs"] = round((wbytes + 2 * xbytes[1]) / (us3 * 1e-6) / 1e9, 1)
        alt["layered_m1_launches_per_step"] = len(stages)
        del g3
        api.bl_check_device_error(stream)

    # ---- end to end through the C ABI with host buffers --------------------
    # Every step copies its bf16 inputs from pinned host memory and its Y back.
    # Two buffer slots and three streams (upload, compute, download) let the
    # copies of one step overlap the kernels of the next, as a serving loop
    # would run them; events order each slot's upload -> compute -> download.
    e2e = None
    if not args.no_e2e:
        h2d = x_all_host.numel() * 2
        d2h = y_all_host.numel() * 4
        n_e2e = max(3, min(steps_timed, 300))
        xa = [x_all, torch.empty_like(x_all)]
        ya = [y_all, torch.empty_like(y_all)]
        yah = [y_all_host, torch.empty_like(y_all_host).pin_memory()]

        def split(buf, lens):
            out, o = {}, 0
            for M in MS:
                out[M] = buf[o:o + lens[M]]
                o += lens[M]
            return out

        xs = [split(b, xlen) for b in xa]
        ys = [split(b, ylen) for b in ya]
        slot_arrs = [{(M, r): fused_problems(M, r, None, xs[k], ys[k]) for M in MS for r in range(R)} for k in range(2)]
        s_up = torch.cuda.Stream(device=dev)
        s_dn = torch.cuda.Stream(device=dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_dn = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize()
        for it in range(n_e2e + 3):
            if it == 3:
                torch.cuda.synchronize()
                t0 = time.perf_counter()
            k = it % 2
            with torch.cuda.stream(s_up):
                s_up.wait_event(ev_comp[k])          # the kernels that read this slot's X are done
                xa[k].copy_(x_all_host, non_blocking=True)
                ev_up[k].record(s_up)
            stream.wait_event(ev_up[k])
            stream.wait_event(ev_dn[k])              # this slot's previous Y has been read back
            for j, M in enumerate(MS):
                rc = L.bl_linear_decode_grouped(slot_arrs[k][(M, replica(it, j))], count, api.BL_BF16, M, 1e-6, RDY, sp)
                if rc:
                    raise api.BitLinearError(rc, "bl_linear_decode_grouped")
            ev_comp[k].record(stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(ev_comp[k])
                yah[k].copy_(ya[k], non_blocking=True)
                ev_dn[k].record(s_dn)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world)
        e2e = {"value": round(world * bytes_step * n_e2e / e2e_s / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "pipelining": "2 buffer slots; one upload and one download per step, on their own streams"}
        api.bl_check_device_error(stream)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": steps_timed,
        "warmup": Wm, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_step": sum(MS), "projections": count,
                   "weight_bytes_per_m": wbytes, "activation_bytes_per_step": sum(2 * xbytes[M] for M in MS),
                   "weight_replicas": R,
                   "l2": f"{R} rotating packed-weight replicas ({R * wbytes / 2**20:.0f} MiB > 3x L2), a different one for every launch",
                   "parallelism": f"replicas x{world}", "launch": "CUDA graph of whole steps, 3 fused launches each"},
        "roofline": roofline, "e2e": e2e, "alt_paths": alt,
        "gpu_launches": steps_timed * len(MS),
    }
    out["clocks"] = clk.summary()
    return out


def prefill(args, dev):
    """Prefill engine on the 1.4B-shape layer (7 projections, M = 8192 tokens):
    int8 TOPS of the contraction (2*M*N*K per projection) for the engine alone
    (bl_forward on pre-quantized inputs) and for the whole per-call path
    (bl_linear: weight quant + act quant + GEMM + rescale)."""
    from ternary_quantized_linear_bitlinear_b200 import api

    items = workloads.prefill1b4()
    M = workloads.PREFILL1B4["tokens"]
    ops = sum(2 * M * W.shape[0] * W.shape[1] for _, W, _ in items)
    dev_items = []
    for name, W, X in items:
        Wd, Xd = W.to(dev), X.to(dev)
        packed, gamma = api.bl_quant_weights(Wd)
        x_q, s = api.bl_quant_act(Xd)
        N, K = W.shape
        Y = torch.empty(M, N, dtype=torch.float32, device=dev)
        ws = torch.empty(api.linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
        dev_items.append((Wd, Xd, packed, gamma, x_q, s, Y, ws))
    L = api.lib()
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream

    def engine():
        for (Wd, Xd, packed, gamma, x_q, s, Y, ws) in dev_items:
            rc = L.bl_forward(packed.data_ptr(), gamma.data_ptr(), x_q.data_ptr(), s.data_ptr(), x_q.shape[0],
                              Y.shape[1], x_q.shape[1], Y.data_ptr(), None, sp)
            if rc:
                raise api.BitLinearError(rc, "bl_forward")

    def whole():
        for (Wd, Xd, packed, gamma, x_q, s, Y, ws) in dev_items:
            rc = L.bl_linear(Wd.data_ptr(), api.BL_BF16, Xd.data_ptr(), api.BL_BF16, Xd.shape[0], Wd.shape[0],
                             Wd.shape[1], None, 1e-6, ws.data_ptr(), ws.numel(), Y.data_ptr(), sp)
            if rc:
                raise api.BitLinearError(rc, "bl_linear")

    # the same layer as four launches: projections sharing an input are one
    # grouped launch (q, k, v | o | gate, up | down)
    names = [n for n, _, _ in items]
    groups = [[names.index(n) for n in g] for g in (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))]
    garrs = []
    for g in groups:
        garr = (api.Problem * len(g))()
        for j, i in enumerate(g):
            (Wd, Xd, packed, gamma, x_q, s, Y, ws) = dev_items[i]
            if j > 0:  # share the first member's activation (the same X in a layer)
                x_q, s = dev_items[g[0]][4], dev_items[g[0]][5]
            garr[j] = api.Problem(packed.data_ptr(), gamma.data_ptr(), x_q.data_ptr(), s.data_ptr(), Y.data_ptr(),
                                  None, Y.shape[1], x_q.shape[1])
        garrs.append((garr, len(g), dev_items[g[0]][4].shape[0]))

    def engine_grouped():
        for garr, n, Mg in garrs:
            rc = L.bl_forward_grouped(garr, n, Mg, 0, sp)
            if rc:
                raise api.BitLinearError(rc, "bl_forward_grouped")

    out = {}
    reps = max(3, min(args.steps, 20))
    for label, fn in (("engine", engine), ("engine_grouped", engine_grouped), ("per_call_quant", whole)):
        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup if args.warmup < 10 else 3)):
                fn()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        out[label] = {"ms_per_layer": round(ms, 4), "tops": round(ops / (ms * 1e-3) / 1e12, 1)}
    # FFN activation + SubLN + act quant feeding the down projection (bl_ffn_act_quant)
    F = workloads.PREFILL1B4["ffn"]
    gate = workloads.normal((M, F), 1.5, 60).to(dev)
    up = workloads.normal((M, F), 1.0, 61).to(dev)
    fgain = workloads.uniform((F,), 0.9, 1.1, 62).to(dev)
    fxq = torch.empty(M, F, dtype=torch.int8, device=dev)
    fs = torch.empty(M, dtype=torch.float32, device=dev)

    def ffn():
        rc = L.bl_ffn_act_quant(gate.data_ptr(), up.data_ptr(), M, F, fgain.data_ptr(), 1e-6, fxq.data_ptr(),
                                fs.data_ptr(), sp)
        if rc:
            raise api.BitLinearError(rc, "bl_ffn_act_quant")

    with torch.cuda.stream(stream):
        for _ in range(3):
            ffn()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(reps):
            ffn()
        f1.record(stream)
    torch.cuda.synchronize()
    ffn_us = f0.elapsed_time(f1) * 1e3 / reps
    ffn_bytes = 2 * M * F * 4 + M * F + 4 * M
    api.bl_check_device_error(stream)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    # int8 dense peak = measured bf16 dense peak x the nominal int8:bf16 ratio (4.5 : 2.25)
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    peak = 2.0 * bf16
    best = "engine_grouped" if out["engine_grouped"]["tops"] >= out["engine"]["tops"] else "engine"
    return {"workload": "prefill1b4: hidden 1536, FFN 4096, q,o 1536^2, k,v 512x1536, gate,up 4096x1536, "
                        "down 1536x4096, M = 8192", "ops_per_layer": ops,
            "engine": out["engine"], "engine_grouped": out["engine_grouped"],
            "engine_grouped_launches": "q,k,v | o | gate,up | down (shared-input projections in one launch)",
            "per_call_quant": out["per_call_quant"],
            "roofline": {"bound": "tensor", "kernel": "k_prefill_tc", "measured_on": best,
                         "achieved": out[best]["tops"],
                         "peak": round(peak, 1), "unit": "TOPS",
                         "peak_source": ("measured bf16 x 2 (nominal int8:bf16)" if "bf16_tflops" in peaks
                                         else "fallback bf16 x 2"),
                         "frac": round(out[best]["tops"] / peak, 4)},
            "ffn_act_quant": {"shape": f"gate, up [{M}, {F}] f32 -> x_q [{M}, {F}] (ReLU^2 gate, SubLN)",
                              "us": round(ffn_us, 2), "gbs": round(ffn_bytes / (ffn_us * 1e-6) / 1e9, 1),
                              "frac_hbm": round(ffn_bytes / (ffn_us * 1e-6) / 1e9 / hbm, 4)},
            "reps": reps, "l2": "inputs and outputs of the layer total > 700 MB"}


def cpu_oracle_step(items_q, wbytes, xbytes):
    """One step of the decode workload on the CPU oracle; returns seconds."""
    import oracle
    t0 = time.perf_counter()
    for M in MS:
        for (wq, g, X) in items_q:
            xq, s = oracle.quant_act(X[:M])
            acc = oracle.contract(xq, wq)
            oracle.rescale(acc, g, s[:, None])
    return time.perf_counter() - t0


def oracle_items(seed=1):
    import numpy as np
    import oracle
    out = []
    for _, W, X in workloads.decode125m(seed=seed, M=max(MS)):
        packed, g, wq = oracle.quant_weights(W.numpy())
        out.append((wq, g, X.float().numpy().astype(np.float32)))
    return out


def cpu_baseline():
    import oracle
    wbytes, xbytes = step_bytes()
    items = oracle_items()
    secs = cpu_oracle_step(items, wbytes, xbytes)
    bytes_step = sum(wbytes + 2 * xbytes[M] for M in MS)
    return {"value": round(bytes_step / secs / 1e9, 4), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "one whole step (84 projections at M = 1, 4, 8: act quant, int64 contraction, rescale); "
                      "OpenMP over token rows"}


def reference(args, rank, world):
    """The CPU oracle as the reference arm, on the same metric and workload;
    each step is one projection (cycling through the 84 and M = 1, 4, 8),
    rows of W subsampled so the run stays within a few minutes."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    items = oracle_items()
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


def main():
    args = parse()
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            out = reference(args, rank, world)
        elif args.mode == "prefill":
            dev = torch.device("cuda", torch.cuda.current_device())
            out = {"mode": "prefill", "prefill": prefill(args, dev)}
        else:
            out = native(args, rank, world, local)
            if args.mode == "all" and rank == 0:
                out["prefill"] = prefill(args, torch.device("cuda", torch.cuda.current_device()))
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline()
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
