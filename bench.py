"""Benchmark of MoE dispatch + combine on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--per-config A,B|none] [--impl ours|reference] [--op OP]

A step is one pass of the whole hot path -- routing metadata, dispatch payload
(bf16 copy or fp8 block quantisation) and combine -- over one batch of
synthetic inputs already resident in HBM.  Steps replay as CUDA graphs that
each hold a rotation of independent input/output sets, so that more than 2x L2
of other data is touched between two uses of the same bytes (or one set alone
is larger than 2x L2); there is no separate L2 flush.  The events bracket the
replays on the launching stream, so they time the GPU work and not Python.

The headline workload is the largest single-GPU batch (T=16384, H=7168, fp8
dispatch with 128-row padding); `per_config` repeats the measurement for the
other T >= 4096 configurations and for the DeepSeek-V3-shaped decode batch.

`value` is the achieved HBM throughput of the step: the algorithmic bytes of
dispatch + combine (x read once, k payload rows written per token, metadata;
combine reads k rows per token and writes y; padding rows are not counted)
divided by the step time, summed over ranks.  Under torchrun every rank runs
its own batch (weak scaling) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_WORKLOAD = "sweep_16384"
PER_CONFIG = ("prefill_zipf", "sweep_4096", "dsv3_decode")
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e specification
B200_L2_BYTES = 126 * 2**20  # nominal; the GPU arm sizes its rotation from the queried L2
METRIC = "dispatch+combine µs and achieved HBM GB/s (% of B200 peak) per config"
FALLBACK_HBM_GBS = 6650.0


def algorithmic_bytes(T, H, E, R, k, fp8):
    """(dispatch bytes, combine bytes) the method must move, padding excluded."""
    S = T * k
    nb = H // 128
    dispatch = T * H * 2 + S * 4 + (S * H + S * nb * 4 if fp8 else S * H * 2)
    dispatch += E * 4 + (E + 1) * 4 + (R + 1) * 4 + 2 * S * 4
    combine = S * H * 2 + 2 * S * 4 + T * H * 2
    return dispatch, combine


def combine_kernel_bytes(T, H, k):
    S = T * k
    return S * H * 2 + 2 * S * 4 + T * H * 2


def measured_peak():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest():
    """Digest of every CUDA source of the library: kernel counters recorded for an
    older digest no longer describe the kernels."""
    d = hashlib.sha256()
    src = os.path.join(HERE, "combine_route_meta_b200", "csrc")
    for name in sorted(os.listdir(src)):
        path = os.path.join(src, name)
        if not os.path.isfile(path):
            continue
        with open(path, "rb") as f:
            d.update(name.encode() + b"\0" + f.read())
    return d.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if the sources are unchanged."""
    p = os.path.join(HERE, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
        if rec["csrc_sha256_16"] != source_digest():
            return None
        return int(rec["bytes_per_launch"][workload][kernel])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons around the timed region.

    Samples arrive every 100 ms; those inside the timed window are used, and if the
    window is shorter than the sampling period, the nearest sample on each side.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []  # (monotonic time, sm_mhz, max_mhz, active reasons)
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            act = [n for n, v in zip(self.REASONS, parts[5:9]) if v.lower().startswith("active")]
            self.samples.append((time.monotonic(), mhz, mx, act))

    def count(self):
        return len(self.samples) if self.proc is not None else 10**9

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()
        if self.proc is not None:
            deadline = time.monotonic() + 1.0
            n = len([s for s in self.samples if s[0] > self.t1])
            while n == 0 and time.monotonic() < deadline:
                time.sleep(0.02)
                n = len([s for s in self.samples if s[0] > self.t1])

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        inside = [s for s in self.samples if self.t0 <= s[0] <= self.t1]
        window = "inside"
        if not inside:
            window = "adjacent"
            before = [s for s in self.samples if s[0] < self.t0][-1:]
            after = [s for s in self.samples if s[0] > self.t1][:1]
            inside = before + after
        if not inside:
            return None
        reasons = sorted({r for s in inside for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": inside[-1][2],
                "reasons": reasons, "samples": len(inside), "window": window}


# ---- CPU oracle arm ---------------------------------------------------------------

def oracle_sample_workload(w):
    """A bounded sample of the workload for the CPU oracle: fewer tokens, same routing recipe."""
    import dataclasses
    t_sample = min(w.T, 512 if w.H >= 4096 else w.T)
    return dataclasses.replace(w, T=t_sample)


class OracleRun:
    """The CPU oracle on a bounded sample of the workload, inputs prepared once."""

    def __init__(self, w):
        import oracle
        from workloads import make_expert_out, make_inputs
        self.oracle = oracle
        oracle.build()
        self.ws = ws = oracle_sample_workload(w)
        _, self.x, self.idx, self.wts = make_inputs(ws)
        self.cap = oracle.rows_capacity(ws.T, ws.k, ws.E, ws.pad128)
        self.eo = None if ws.identity_experts else make_expert_out(ws, self.cap)
        db, cb = algorithmic_bytes(ws.T, ws.H, ws.E, ws.R, ws.k, ws.fp8)
        self.bytes = db + cb
        self.desc = (f"oracle dispatch+combine (single-threaded C, fp64 combine) on the first "
                     f"{ws.T} of {w.T} tokens of {w.name}")

    def once(self):
        """Seconds for one dispatch + combine."""
        ws, o = self.ws, self.oracle
        t0 = time.perf_counter()
        d = o.dispatch(self.x, self.idx, E=ws.E, R=ws.R, fp8=ws.fp8, pad128=ws.pad128,
                       rows_cap=self.cap)
        o.combine(d["slot"], self.wts, d["recv_x"] if self.eo is None else self.eo)
        return time.perf_counter() - t0


class OracleRunParallel(OracleRun):
    """The same oracle on the same sample, its payload and combine split over
    every host core by token range (the layout stays one serial walk)."""

    def __init__(self, w, threads):
        super().__init__(w)
        self.threads = threads
        self.desc = (f"oracle dispatch+combine (C, fp64 combine; payload and combine split by "
                     f"token range over {threads} host threads) on the first {self.ws.T} of "
                     f"{w.T} tokens of {w.name}")

    def once(self):
        ws, o = self.ws, self.oracle
        t0 = time.perf_counter()
        d = o.dispatch_parallel(self.x, self.idx, E=ws.E, R=ws.R, fp8=ws.fp8, pad128=ws.pad128,
                                rows_cap=self.cap, threads=self.threads)
        o.combine_parallel(d["slot"], self.wts, d["recv_x"] if self.eo is None else self.eo, self.threads)
        return time.perf_counter() - t0


def time_oracle(w, budget_s=10.0, max_reps=50, threads=None):
    """(GB/s of algorithmic bytes, description) of the oracle on a bounded sample
    (on `threads` host threads when given)."""
    run = OracleRun(w) if threads is None else OracleRunParallel(w, threads)
    times = []
    t_end = time.perf_counter() + budget_s
    while len(times) < max_reps and (not times or time.perf_counter() < t_end):
        times.append(run.once())
    med = statistics.median(times)
    return run.bytes / med / 1e9, f"{run.desc}, median of {len(times)} runs"


# ---- GPU arm ----------------------------------------------------------------------------

def max_over_ranks(value, dist, device):
    """The largest of every rank's value (all ranks take part and all get it)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(step_bytes, world, ms_per_step):
    """Whole-job GB/s: every rank moves step_bytes per step (weak scaling)."""
    return step_bytes * world / (ms_per_step * 1e-3) / 1e9


def graph_kernels(g):
    """Names of the kernel nodes in a captured torch CUDA graph (one replay's launches)."""
    from cuda.bindings import driver as drv
    graph = drv.CUgraph(g.raw_cuda_graph())
    err, _, n = drv.cuGraphGetNodes(graph, 0)
    if err != drv.CUresult.CUDA_SUCCESS:
        raise RuntimeError(f"cuGraphGetNodes: {err}")
    err, nodes, n = drv.cuGraphGetNodes(graph, n)
    names = []
    for node in nodes[:n]:
        err, kind = drv.cuGraphNodeGetType(node)
        if kind != drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
            continue
        name = "?"
        try:
            err, params = drv.cuGraphKernelNodeGetParams(node)
            err, raw = drv.cuFuncGetName(params.func)
            name = raw.decode() if isinstance(raw, bytes) else str(raw)
        except Exception:
            pass
        names.append(name)
    return names


def short_kernel_name(mangled):
    for k in ("dispatch_fused", "dispatch_direct", "dispatch_multi", "scatter_bulk_bf16",
              "scatter_bulk_fp8", "scatter_rows", "combine_rows", "meta_single_block", "meta_tile_count",
              "meta_tile_scan", "meta_tile_assign"):
        if k in mangled:
            return k
    return mangled


def step_set_bytes(w, rows_cap):
    """Bytes one step's input/output set occupies on the device."""
    S = w.T * w.k
    recv = rows_cap * w.H * (1 if w.fp8 else 2) + (rows_cap * (w.H // 128) * 4 if w.fp8 else 0)
    eo = 0 if w.identity_experts else rows_cap * w.H * 2
    return (w.T * w.H * 2 + S * 4 + S * 4 + eo + recv + rows_cap * 4 + S * 4 + w.T * w.H * 2)


def rotating_sets(set_bytes, l2_bytes):
    """Independent input/output sets to rotate through, so that more than 2x L2
    of other sets' bytes is touched before a set is used again (1: one set is
    already larger than 2x L2)."""
    import math
    return 1 if set_bytes >= 2 * l2_bytes else min(64, math.ceil(2 * l2_bytes / set_bytes) + 1)


def config_for(w, world, rows_cap, parallelism="replicas"):
    """The `config` object of a JSON line; both arms print the same one."""
    one_set = rotating_sets(step_set_bytes(w, rows_cap), B200_L2_BYTES) == 1
    return {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "R": w.R, "k": w.k,
            "payload": "fp8 e4m3 + fp32 scale per 128" if w.fp8 else "bf16",
            "pad128": w.pad128, "combine": "bf16 out, fp32 accumulate",
            "l2": ("inputs larger than 2x L2 every step (no flush needed)" if one_set else
                   "rotating input sets: over 2x L2 of other sets touched between uses of a set"),
            "graphs": ("CUDA graphs of 8+ steps over the rotating sets, replayed back to back"
                       if parallelism == "replicas" else "one step per CUDA graph replay"),
            "inputs": "written before the step; the dispatch is told so (MOE_INPUTS_READY)",
            "parallelism": f"{parallelism} x{world}"}


def run_gpu(args, name, rank, world, with_e2e):
    """Times K steps of one workload on this rank's GPU; returns the raw figures."""
    import dataclasses

    import torch
    import combine_route_meta_b200 as moe
    from workloads import WORKLOADS, make_expert_out, make_inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = dataclasses.replace(WORKLOADS[name], seed=WORKLOADS[name].seed + rank)
    if w.identity_experts and w.fp8:
        raise SystemExit("identity experts need a bf16 dispatch")
    _, x, idx, wts = make_inputs(w)
    # Every step's inputs were written before the kernel ahead of its dispatch
    # (that kernel is the previous step's combine, or in the end-to-end loop the
    # inputs arrive by host copies): MOE_INPUTS_READY holds.
    cfg = moe.make_config(w.H, w.k, w.E, w.R, w.fp8, w.pad128, inputs_ready=True)
    rows_cap = moe.rows_capacity(cfg, w.T)
    eo_host = None if w.identity_experts else make_expert_out(w, rows_cap)

    def bf16_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    # Inputs larger than L2 between uses of the same bytes: rotate through enough
    # independent sets (inputs and outputs) that one step's data is evicted
    # before it comes round again.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = step_set_bytes(w, rows_cap)
    nsets = rotating_sets(set_bytes, l2)

    class Set:
        pass

    sets = []
    for _ in range(nsets):
        st = Set()
        st.buf = moe.Buffers(cfg, w.T, dev)
        st.x, st.idx, st.w = bf16_dev(x), torch.from_numpy(idx).to(dev), torch.from_numpy(wts).to(dev)
        st.eo = st.buf.recv_x if eo_host is None else bf16_dev(eo_host)
        st.y = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
        sets.append(st)
    stream = torch.cuda.Stream(device=dev)

    def do_dispatch(st):
        moe.dispatch_into(st.buf, st.x, st.idx, st.w, stream=stream)

    def do_combine(st):
        moe.combine_into(st.buf.handle_c, st.eo, st.y, st.buf.err, stream=stream)

    with torch.cuda.stream(stream):
        for st in sets:
            do_dispatch(st)
            do_combine(st)
    stream.synchronize()
    if moe.check(stream) != 0:
        raise RuntimeError("device error during warm-up")

    # CUDA graphs.  A top-level submission (a kernel launch or a graph launch)
    # costs about 2 us on this GPU however small its work, while a kernel
    # boundary inside a graph costs well under 1 us; a serving engine captures a
    # whole forward pass.  So one graph holds a rotation of steps, one per input
    # set (a step = dispatch + combine on that set), and K steps are replayed as
    # whole rotations plus one graph with the remainder.
    def capture(fns):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g, stream=stream):
            for fn in fns:
                fn()
        return g

    def rotation(make, count):
        return capture([make(sets[i % nsets]) for i in range(count)])

    step_fn = lambda st: (lambda: (do_dispatch(st), do_combine(st)))
    disp_fn = lambda st: (lambda: do_dispatch(st))
    comb_fn = lambda st: (lambda: do_combine(st))
    pay_fn = lambda st: (lambda: moe.dispatch_payload_into(st.buf, st.x, stream=stream))

    g_one = rotation(step_fn, 1)
    step_kernels = [short_kernel_name(k) for k in graph_kernels(g_one)]
    disp_kernels = [short_kernel_name(k) for k in graph_kernels(rotation(disp_fn, 1))]
    del g_one
    launches_per_step = len(step_kernels)
    graph_cache = {}

    per_graph = max(nsets, 8)

    def graphs_for(gname, make, n):
        """(full-rotation graph, remainder graph or None, rotations) covering n steps."""
        q, r = divmod(n, per_graph)
        key = (gname, r)
        if key not in graph_cache:
            full = rotation(make, per_graph)
            full.instantiate()
            rest = None
            if r:
                rest = rotation(make, r)
                rest.instantiate()
            graph_cache[key] = (full, rest)
        full, rest = graph_cache[key]
        return full, rest, q

    def run(gname, make, n, per_replay=False):
        """Runs n steps of `make` back to back (rotating sets).  Returns device
        milliseconds, and with per_replay the milliseconds per step of each
        full-rotation replay."""
        full, rest, q = graphs_for(gname, make, n)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range((q if per_replay else 0) + 2)]
        with torch.cuda.stream(stream):
            # a sleeping kernel in front lets the host queue the replays ahead of the GPU
            torch.cuda._sleep(min(q + 1, 256) * 100_000)
            ev[0].record(stream)
            for i in range(q):
                full.replay()
                if per_replay:
                    ev[i + 1].record(stream)
            if rest is not None:
                rest.replay()
            ev[-1].record(stream)
        ev[-1].synchronize()
        total = ev[0].elapsed_time(ev[-1])
        if not per_replay:
            return total
        return total, [ev[i].elapsed_time(ev[i + 1]) / per_graph for i in range(q)]

    # Warm-up: at least W steps, and on until the clock sampler reports (the GPU
    # is then under load when the timed region starts).
    sampler = ClockSampler(dev.index)
    sampler.start()
    t_warm = time.monotonic()
    run("step", step_fn, max(args.warmup, per_graph))
    while sampler.count() < 3 and time.monotonic() - t_warm < 5.0:
        run("step", step_fn, 20 * per_graph)
    graphs_for("step", step_fn, args.steps)  # capture before the timed region
    torch.cuda.synchronize()

    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_start()
    total_ms = run("step", step_fn, args.steps)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_end()
    clocks = sampler.stop()
    bits = moe.check(stream)
    if bits:
        raise RuntimeError(f"device error bits {bits} during timing")
    if dist is not None:
        total_ms = max_over_ranks(total_ms, dist, dev)

    # Spread: the same K steps again with an event after every full-rotation
    # replay (the events add a little time, so the headline is the pass above).
    _, per_step_ms = run("step", step_fn, args.steps, per_replay=True)

    # Phase split, same protocol: K dispatches alone, K combines alone, and on the
    # multi-kernel dispatch path K payload kernels alone (moe_dispatch_payload on
    # the slots the last dispatch of each set left).
    disp_ms = run("disp", disp_fn, args.steps)
    comb_ms = run("comb", comb_fn, args.steps)
    pay_ms = run("pay", pay_fn, args.steps) if len(disp_kernels) > 1 else None
    if dist is not None:
        disp_ms = max_over_ranks(disp_ms, dist, dev)
        comb_ms = max_over_ranks(comb_ms, dist, dev)
        if pay_ms is not None:
            pay_ms = max_over_ranks(pay_ms, dist, dev)
    graph_cache.clear()

    e2e = None
    if with_e2e:
        # End to end through the public API with host buffers, every step: H2D
        # of the step's inputs from pinned memory, dispatch, combine, D2H of y.
        # Steady state of a stream of batches: two device sets, the uploads on
        # one copy stream and the downloads on another, so step i's result goes
        # down while step i+1's inputs come up (the host link is full duplex)
        # and the kernels run between them.  Events order the reuse of a set.
        pin = dict(pin_memory=True)
        x_h = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
        idx_h = torch.from_numpy(idx).pin_memory()
        w_h = torch.from_numpy(wts).pin_memory()
        eo_h = (None if eo_host is None else
                torch.from_numpy(np.ascontiguousarray(eo_host).view(np.int16)).view(torch.bfloat16).pin_memory())
        pipe = [sets[0]]
        if len(sets) > 1:
            pipe.append(sets[1])
        else:
            st2 = Set()
            st2.buf = moe.Buffers(cfg, w.T, dev)
            st2.x, st2.idx, st2.w = torch.empty_like(sets[0].x), torch.empty_like(sets[0].idx), \
                torch.empty_like(sets[0].w)
            st2.eo = st2.buf.recv_x if eo_host is None else torch.empty_like(sets[0].eo)
            st2.y = torch.empty_like(sets[0].y)
            pipe.append(st2)
        y_h = [torch.empty((w.T, w.H), dtype=torch.bfloat16, **pin) for _ in pipe]
        h2d = x_h.numel() * 2 + idx_h.numel() * 4 + w_h.numel() * 4 + (0 if eo_h is None else eo_h.numel() * 2)
        d2h = y_h[0].numel() * 2
        s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up_done = [torch.cuda.Event() for _ in pipe]
        comp_done = [torch.cuda.Event() for _ in pipe]
        down_done = [torch.cuda.Event() for _ in pipe]
        for b in range(len(pipe)):  # every event recorded once before its first wait
            for ev in (up_done[b], comp_done[b], down_done[b]):
                ev.record(stream)

        def e2e_step(i):
            b = i % len(pipe)
            st = pipe[b]
            with torch.cuda.stream(s_up):
                s_up.wait_event(comp_done[b])     # the set's previous step has read its inputs
                st.x.copy_(x_h, non_blocking=True)
                st.idx.copy_(idx_h, non_blocking=True)
                st.w.copy_(w_h, non_blocking=True)
                if eo_h is not None:
                    st.eo.copy_(eo_h, non_blocking=True)
                up_done[b].record(s_up)
            stream.wait_event(up_done[b])
            stream.wait_event(down_done[b])       # the set's previous y has gone down
            do_dispatch(st)
            do_combine(st)
            comp_done[b].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[b])
                y_h[b].copy_(st.y, non_blocking=True)
                down_done[b].record(s_down)

        e2e_steps = max(3, min(args.steps, 20))
        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()  # every rank's copies share the node's host links while timed
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        for i in range(e2e_steps):
            e2e_step(args.warmup + i)
        s_down.wait_stream(s_up)
        s_down.wait_stream(stream)
        e1.record(s_down)
        e1.synchronize()
        e2e_med_ms = e0.elapsed_time(e1) / e2e_steps
        if dist is not None:
            e2e_med_ms = max_over_ranks(e2e_med_ms, dist, dev)
        torch.cuda.synchronize()
        if moe.check(stream) != 0:
            raise RuntimeError("device error during the end-to-end steps")
        e2e = dict(ms=e2e_med_ms, h2d=h2d, d2h=d2h)
        del pipe

    sets.clear()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return dict(w=w, rows_cap=rows_cap, total_ms=total_ms, per_step_ms=per_step_ms, disp_ms=disp_ms,
                comb_ms=comb_ms, pay_ms=pay_ms, clocks=clocks, launches_per_step=launches_per_step,
                step_kernels=step_kernels, disp_kernels=disp_kernels, e2e=e2e, nsets=nsets,
                set_bytes=set_bytes, l2=l2, per_graph=per_graph)


def ep_ranks_check(E, world):
    """Expert parallelism puts E/world experts on each rank: world must divide E
    and stay within the library's rank limit."""
    if world < 1 or E % world != 0 or world > 64:
        raise SystemExit(f"--parallelism ep: {world} ranks cannot share {E} experts evenly (at most 64)")


def ep_step_bytes(w):
    """Algorithmic bytes of one rank's expert-parallel step: its dispatch and
    combine, as on one GPU (x read once, k rows written, k rows read back, y
    written, and the metadata); the rows cross NVLink or stay local depending
    on which rank hosts the expert."""
    d, c = algorithmic_bytes(w.T, w.H, w.E, 1, w.k, w.fp8)
    return d + c


def run_ep(args, name, rank, world):
    """Expert parallelism over `world` GPUs, one rank each: every rank
    dispatches its own batch to the ranks hosting its experts and combines their
    outputs (ExpertParallel: NCCL count exchange, peer stores, device-side
    completion flags).  Returns the max-over-ranks device milliseconds of K steps."""
    import dataclasses
    import datetime

    import torch
    import torch.distributed as dist
    import combine_route_meta_b200 as moe
    from combine_route_meta_b200.ep import ExpertParallel
    from workloads import WORKLOADS, make_expert_out, make_inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    if not dist.is_initialized():   # one rank without torchrun
        import socket
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
    w = dataclasses.replace(WORKLOADS[name], seed=WORKLOADS[name].seed + rank)
    ep_ranks_check(w.E, world)
    _, x, idx, wts = make_inputs(w)
    ep = ExpertParallel(w.H, w.k, w.E, w.fp8, w.pad128, T_max=w.T, device=dev)
    ep.expert_out.copy_(torch.from_numpy(np.ascontiguousarray(make_expert_out(w, ep.rows_cap)).view(np.int16))
                        .to(dev).view(torch.bfloat16))
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)
    idd, wd = torch.from_numpy(idx).to(dev), torch.from_numpy(wts).to(dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        dst = ep.dispatch(xd, idd, stream)
        ep.experts_done(stream)     # the experts' kernels would run here
        return ep.combine(idd, dst, wd, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    ep.check(stream)
    # one step as a CUDA graph (every rank captures the same collective and
    # kernels), replayed once per step
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    sampler = ClockSampler(dev.index)
    sampler.start()
    t_warm = time.monotonic()
    while sampler.count() < 3 and time.monotonic() - t_warm < 5.0:
        with torch.cuda.stream(stream):
            for _ in range(20):
                g.replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_end()
    clocks = sampler.stop()
    ep.check(stream)
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    kernels_per_step = 7   # layout, rows, payload, wait, signal, wait, combine (and the NCCL all-gather)
    del g   # a graph holding NCCL work is released before the group is destroyed
    del ep
    return dict(w=w, total_ms=ms, clocks=clocks, kernels_per_step=kernels_per_step)


def summarize(r, steps, world, peak, peak_kind):
    """The per-workload figures of a JSON line: throughput, phase times, the
    per-kernel rooflines and the clocks."""
    w = r["w"]
    db, cb = algorithmic_bytes(w.T, w.H, w.E, w.R, w.k, w.fp8)
    step_bytes = db + cb
    ms_per_step = r["total_ms"] / steps
    value = job_throughput(step_bytes, world, ms_per_step)
    disp_us = r["disp_ms"] / steps * 1e3
    comb_us = r["comb_ms"] / steps * 1e3
    # Per-kernel rooflines: the dispatch payload kernel (the fused kernel on the
    # one-launch path) and the combine kernel, each timed alone over K launches.
    S = w.T * w.k
    kernels = []
    if r["pay_ms"] is None:
        kernels.append((r["disp_kernels"][0], db, disp_us))
    else:
        name = ([k for k in r["disp_kernels"] if k.startswith("scatter")] or ["payload"])[-1]
        pay_bytes = (w.T * w.H * 2 + S * 4
                     + (S * w.H + S * (w.H // 128) * 4 if w.fp8 else S * w.H * 2))
        kernels.append((name, pay_bytes, r["pay_ms"] / steps * 1e3))
    kernels.append(("combine_rows", combine_kernel_bytes(w.T, w.H, w.k), comb_us))
    per_kernel = []
    for name, nbytes, us in kernels:
        gbs = nbytes / (us * 1e-6) / 1e9
        per_kernel.append({"kernel": name, "us": round(us, 3), "algorithmic_bytes": nbytes,
                           "achieved": round(gbs, 1), "frac": round(gbs / peak, 4),
                           "traffic": recorded_traffic(name, w.name)})
    dom = max(per_kernel, key=lambda k: k["us"])
    roofline = {"bound": "hbm", "kernel": dom["kernel"], "achieved": dom["achieved"],
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": dom["frac"],
                "traffic": dom["traffic"], "algorithmic_bytes": dom["algorithmic_bytes"],
                "kernels": per_kernel}
    ps = sorted(r["per_step_ms"])
    pct = lambda p: round(ps[min(len(ps) - 1, int(p * len(ps)))] * 1e3, 3) if ps else None
    return {
        "value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms_per_step, 5),
        "dispatch_us": round(disp_us, 2), "combine_us": round(comb_us, 2),
        "total_us": round(ms_per_step * 1e3, 2),
        "pct_of_peak": round(100 * step_bytes / (ms_per_step * 1e-3) / 1e9 / peak, 2),
        "pct_of_spec_peak": round(100 * step_bytes / (ms_per_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 2),
        "bytes_per_step": {"dispatch": db, "combine": cb},
        "step_us_spread": {"p10": pct(0.1), "p50": pct(0.5), "p90": pct(0.9), "replays": len(ps),
                           "steps_per_replay": r["per_graph"]},
        "roofline": roofline,
        "kernels_per_step": r["step_kernels"],
        "timing": {"sets": r["nsets"], "set_bytes": r["set_bytes"], "l2_bytes": r["l2"],
                   "steps_per_graph": r["per_graph"]},
        "clocks": r["clocks"],
    }


# ---- the rows next to the hot path: one kernel at a time ---------------------------

EXPERT_INTERMEDIATE = 2048  # DeepSeek-V3 / Kimi-K2 routed-expert intermediate size


def partial_accuracy(moe, d, wts, b, w, dev, sample=64):
    """Errors of sender-side (per-rank partial) and receiver-only combine against
    the fp64 weighted sum, on a sample of tokens: max and mean absolute error,
    and the share of outputs where the two bf16 results differ."""
    import torch
    y_send = b["y"].view(torch.int16).cpu().numpy().view(np.uint16)
    y_recv = moe.combine(d.handle, b["eo"]).view(torch.int16).cpu().numpy().view(np.uint16)
    slot = d.handle.slot.cpu().numpy()
    toks = np.linspace(0, w.T - 1, min(sample, w.T)).astype(np.int64)
    to_f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    sl = slot[toks]                                     # [n, k]
    rows = torch.from_numpy(np.maximum(sl, 0).reshape(-1)).to(dev)
    v = to_f(b["eo"].view(torch.int16)[rows].cpu().numpy().view(np.uint16)).reshape(len(toks), w.k, w.H)
    wk = np.where(sl >= 0, wts[toks].astype(np.float64), 0.0)
    exact = np.einsum("nk,nkh->nh", wk, v)
    out = {}
    for name, y in (("receiver", y_recv), ("sender", y_send)):
        err = np.abs(to_f(y[toks]) - exact)
        out[name] = {"max_abs": float(err.max()), "mean_abs": float(err.mean())}
    out["differ_frac"] = float(np.mean(y_send[toks] != y_recv[toks]))
    out["tokens"] = int(len(toks))
    return out


def run_op(args, peak, peak_kind):
    """Times one next-row kernel on a workload's shapes; prints one JSON line."""
    import dataclasses
    import math
    import torch
    import combine_route_meta_b200 as moe
    from workloads import WORKLOADS, make_expert_out, make_inputs, normal_bf16_rows

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    _, x, idx, wts = make_inputs(w)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)

    def bf16_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    d = moe.dispatch(bf16_dev(x), torch.from_numpy(idx).to(dev), torch.from_numpy(wts).to(dev),
                     w.E, w.R, w.fp8, w.pad128)
    rows = d.recv_x.shape[0]
    S = w.T * w.k
    if args.op == "rank_partial":
        eo = bf16_dev(make_expert_out(w, rows))
        set_bytes = rows * w.H * 2 + 2 * S * w.H * 2
        make = lambda: dict(partial=torch.empty((w.T, w.k, w.H), dtype=torch.bfloat16, device=dev),
                            prank=torch.empty((w.T, w.k), dtype=torch.int32, device=dev),
                            npart=torch.empty(w.T, dtype=torch.int32, device=dev),
                            y=torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev), eo=eo.clone())
        fn = lambda b: (lambda: moe.combine_rank_partial_into(
            d.handle.c, d.rank_offset, b["eo"], b["partial"], b["prank"], b["npart"], b["y"],
            moe.error_word(dev), stream))
    elif args.op == "silu_quant":
        I = EXPERT_INTERMEDIATE
        gu = bf16_dev(normal_bf16_rows(w.seed, 9, 0, rows, 2 * I))
        set_bytes = rows * (4 * I + I + I // 32)
        make = lambda: dict(gu=gu.clone(), act=torch.empty((rows, I), dtype=torch.float8_e4m3fn, device=dev),
                            sc=torch.empty((rows, I // 128), dtype=torch.float32, device=dev))
        fn = lambda b: (lambda: moe.silu_quant_into(b["gu"], d.recv_src, d.expert_offset[w.E:],
                                                    b["act"], b["sc"], False, stream))
    elif args.op == "router":
        logits = torch.from_numpy(np.random.default_rng(w.seed).standard_normal((w.T, w.E)).astype(np.float32)).to(dev)
        set_bytes = w.T * w.E * 4 + S * 8
        make = lambda: dict(l=logits.clone(), idx=torch.empty((w.T, w.k), dtype=torch.int32, device=dev),
                            w=torch.empty((w.T, w.k), dtype=torch.float32, device=dev))
        fn = lambda b: (lambda: moe.router_topk_into(b["l"], w.k, b["idx"], b["w"],
                                                     score_fn="sigmoid" if w.routing == "sigmoid_topk" else "softmax",
                                                     stream=stream))
    elif args.op == "route_dispatch":
        logits = torch.from_numpy(np.random.default_rng(w.seed).standard_normal((w.T, w.E)).astype(np.float32)).to(dev)
        cfg = moe.make_config(w.H, w.k, w.E, w.R, w.fp8, w.pad128)
        x_dev = bf16_dev(x)
        set_bytes = w.T * w.E * 4 + sum(algorithmic_bytes(w.T, w.H, w.E, w.R, w.k, w.fp8)[:1])
        make = lambda: dict(l=logits.clone(), x=x_dev.clone(), buf=moe.Buffers(cfg, w.T, dev),
                            idx=torch.empty((w.T, w.k), dtype=torch.int32, device=dev),
                            w=torch.empty((w.T, w.k), dtype=torch.float32, device=dev))
        fn = lambda b: (lambda: moe.route_dispatch_into(
            b["buf"], b["x"], b["l"], b["idx"], b["w"],
            score_fn="sigmoid" if w.routing == "sigmoid_topk" else "softmax", stream=stream))
    elif args.op == "ep":
        # W = the workload's R virtual ranks on this GPU, each with the workload's
        # batch (its own routing seed); one launch = every rank's local layout,
        # rows, payload and combine, the count exchange being each rank's
        # counts written into its row of counts_all.  All buffers are local, so
        # this times the kernels against HBM, not NVLink.
        import ctypes
        W = w.R
        ranks = [make_inputs(dataclasses.replace(w, seed=w.seed + 101 * r)) for r in range(W)]
        cfg = moe.make_config(w.H, w.k, w.E, W, w.fp8, w.pad128)
        cfg1 = moe.make_config(w.H, w.k, w.E, 1, False, False)
        cap = moe.ep_rows_capacity(cfg, w.T)
        nws = moe.workspace_bytes(cfg1, w.T)
        i32 = dict(dtype=torch.int32, device=dev)
        fp8_dt = torch.float8_e4m3fn if w.fp8 else torch.bfloat16
        set_bytes = W * cap * (w.H * (1 if w.fp8 else 2) + w.H * 2)
        # every rank's buffers hold the worst case (all entries to one rank), so
        # many ranks with long batches would need far more memory than the GPU
        # or the host generator can give; refuse those before allocating
        if set_bytes > 8 << 30:
            raise SystemExit(f"--op ep: {W} ranks x {cap} rows of worst-case buffers need "
                             f"{set_bytes / 2**30:.0f} GiB; use a workload with fewer ranks or tokens")
        def make():
            b = dict(counts=torch.empty((W, w.E), **i32), eo=[], recv_x=[], recv_sc=[], r=[])
            for r in range(W):
                _, xr, ir, wr = ranks[r]
                b["recv_x"].append(torch.empty((cap, w.H), dtype=fp8_dt, device=dev))
                b["recv_sc"].append(torch.empty((cap, w.H // 128), dtype=torch.float32, device=dev)
                                    if w.fp8 else None)
                b["eo"].append(bf16_dev(normal_bf16_rows(w.seed + r, 3, 0, cap, w.H)))
                rr = dict(x=bf16_dev(xr), idx=torch.from_numpy(ir).to(dev), w=torch.from_numpy(wr).to(dev),
                          off=torch.empty(w.E + 1, **i32), roff=torch.empty(2, **i32),
                          src=torch.empty(S, **i32), slot=torch.empty((w.T, w.k), **i32),
                          ws=torch.empty(max(nws, 1), dtype=torch.uint8, device=dev),
                          dst=torch.empty((w.T, w.k), **i32), rc=torch.empty(w.E // W, **i32),
                          ro=torch.empty(w.E // W + 1, **i32),
                          y=torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev))
                rr["out"] = moe.moe_dispatch_out(None, None, b["counts"][r].data_ptr(), rr["off"].data_ptr(),
                                                 rr["roff"].data_ptr(), rr["src"].data_ptr(), S)
                # completion state: "rows" and "outputs" flags, epochs, CTA count
                rr["fl_rows"], rr["fl_out"] = torch.zeros(W, **i32), torch.zeros(W, **i32)
                rr["epochs"], rr["done"] = torch.zeros(2, **i32), torch.zeros(1, **i32)
                b["r"].append(rr)
            b["fl_rows"] = [rr["fl_rows"] for rr in b["r"]]
            b["fl_out"] = [rr["fl_out"] for rr in b["r"]]
            return b
        def ep_step(b):
            P = ctypes.c_void_p
            err = moe.error_word(dev)
            for rr in b["r"]:
                moe._ok(moe.moe_dispatch_layout(ctypes.byref(cfg1), w.T, P(rr["idx"].data_ptr()),
                                                ctypes.byref(rr["out"]), P(rr["slot"].data_ptr()),
                                                P(rr["ws"].data_ptr()), nws, P(err.data_ptr()),
                                                P(stream.cuda_stream)), "layout")
            for r, rr in enumerate(b["r"]):
                moe.ep_layout_into(cfg, r, rr["idx"], rr["slot"], rr["off"], b["counts"], cap, rr["dst"],
                                   rr["rc"], rr["ro"], err, stream)
                moe.ep_dispatch_payload_into(cfg, rr["x"], rr["idx"], rr["dst"], b["recv_x"],
                                             b["recv_sc"] if w.fp8 else None, cap, err, stream,
                                             signal=(r, b["fl_rows"], rr["epochs"][0:1], rr["done"]))
            for rr in b["r"]:
                moe.ep_wait_into(rr["fl_rows"], rr["epochs"][0:1], 1_000_000_000, err, stream)
            for r, rr in enumerate(b["r"]):
                moe.ep_signal_into(r, b["fl_out"], rr["epochs"][1:2], stream)
            for rr in b["r"]:
                moe.ep_wait_into(rr["fl_out"], rr["epochs"][1:2], 1_000_000_000, err, stream)
                moe.ep_combine_into(cfg, rr["idx"], rr["dst"], rr["w"], b["eo"], cap, rr["y"], err, stream)
        fn = lambda b: (lambda: ep_step(b))
    else:
        raise SystemExit(f"unknown --op {args.op}")
    nsets = 1 if set_bytes >= 2 * l2 else min(64, math.ceil(2 * l2 / set_bytes) + 1)
    sets = [make() for _ in range(nsets)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for b in sets:
            fn(b)()
    stream.synchronize()
    per_graph = max(nsets, 8)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(per_graph):
            fn(sets[i % nsets])()
    reps = max(1, args.steps // per_graph)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for timed in (False, True):
        with torch.cuda.stream(stream):
            torch.cuda._sleep(min(reps, 256) * 100_000)
            e0.record(stream)
            for _ in range(reps if timed else max(1, args.warmup // per_graph)):
                g.replay()
            e1.record(stream)
        e1.synchronize()
    launches = reps * per_graph
    us = e0.elapsed_time(e1) * 1e3 / launches
    if moe.check(stream):
        raise RuntimeError("device error bits during timing")
    # algorithmic bytes of one launch
    if args.op == "rank_partial":
        npart = int(sets[0]["npart"].sum().item())
        nbytes = S * w.H * 2 + 2 * S * 4 + (w.R + 1) * 4 + 2 * npart * w.H * 2 + w.T * 4 + w.T * w.H * 2
        extra = {"partials": npart, "accuracy": partial_accuracy(moe, d, wts, sets[0], w, dev)}
    elif args.op == "silu_quant":
        used = int((d.recv_src >= 0).sum().item())
        I = EXPERT_INTERMEDIATE
        nbytes = used * (4 * I + I + (I // 128) * 4) + used * 4
        extra = {"rows_used": used, "I": I}
    elif args.op == "route_dispatch":
        nbytes = w.T * w.E * 4 + S * 8 + algorithmic_bytes(w.T, w.H, w.E, w.R, w.k, w.fp8)[0]
        extra = {}
    elif args.op == "ep":
        nbytes = sum(algorithmic_bytes(w.T * w.R, w.H, w.E, w.R, w.k, w.fp8))
        extra = {"ranks": w.R, "tokens_per_rank": w.T, "kernels_per_launch": 7 * w.R,
                 "note": "virtual ranks on one GPU: local buffers, HBM-bound, no NVLink"}
    else:
        nbytes = w.T * w.E * 4 + S * 8
        extra = {}
    gbs = nbytes / (us * 1e-6) / 1e9
    op_kernels = {"rank_partial": ["combine_partial_send", "combine_partial_recv"],
                  "silu_quant": ["silu_quant_rows"], "router": ["router_topk"],
                  "ep": ["ep_rows", "ep_payload", "ep_combine"],
                  "route_dispatch": ["router_topk", "dispatch_direct", "dispatch_fused", "dispatch_multi",
                                     "scatter_rows", "scatter_bulk_bf16", "scatter_bulk_fp8"]}[args.op]
    extra["traffic"] = {k: recorded_traffic(k, w.name) for k in op_kernels}
    line = {"op": args.op, "workload": w.name, "us": round(us, 3), "algorithmic_bytes": nbytes,
            "achieved_GBs": round(gbs, 1), "peak": peak, "peak_kind": peak_kind,
            "frac": round(gbs / peak, 4), "launches_timed": launches,
            "l2": f"{nsets} rotating sets of {set_bytes / 1e6:.1f} MB", **extra}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--per-config", default=None,
                    help="comma-separated workloads measured after the headline one and reported "
                         "under per_config (default: the other T >= 4096 configs and the decode "
                         "config when the headline is the default; 'none' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parallelism", default="replicas", choices=["replicas", "ep"],
                    help="replicas: every rank runs its own single-GPU step; ep: the ranks form one "
                         "expert-parallel group (rank d hosts experts [d E/N, (d+1) E/N))")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default=None, choices=["rank_partial", "silu_quant", "router", "route_dispatch",
                                                   "ep"],
                    help="time one of the kernels next to the hot path instead of the step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    from workloads import WORKLOADS
    if args.workload not in WORKLOADS:
        ap.error(f"unknown workload {args.workload}")
    w0 = WORKLOADS[args.workload]
    peak, peak_kind = measured_peak()
    if args.per_config is None:
        per_config = list(PER_CONFIG) if args.workload == DEFAULT_WORKLOAD else []
    elif args.per_config.strip().lower() in ("", "none"):
        per_config = []
    else:
        per_config = [p.strip() for p in args.per_config.split(",") if p.strip()]
    for p in per_config:
        if p not in WORKLOADS:
            ap.error(f"unknown workload {p} in --per-config")

    if args.op is not None:
        run_op(args, peak, peak_kind)
        return

    if args.impl == "reference":
        # The reference arm is the CPU oracle, timed on this host's cores (rank 0 only).
        if rank != 0:
            return
        import oracle
        run = OracleRun(w0)
        per_step = [run.once() for _ in range(args.warmup + args.steps)][args.warmup:]
        total = sum(per_step)
        g = run.bytes * args.steps / total / 1e9
        ms = total / args.steps * 1e3
        desc = f"{run.desc}, {args.steps} timed runs"
        cap = oracle.rows_capacity(w0.T, w0.k, w0.E, w0.pad128)
        line = {
            "impl": "reference", "metric": METRIC, "value": round(g, 3), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(w0, max(world, args.gpus), cap if args.parallelism == "replicas" else w0.T * w0.k,
                                 args.parallelism),
            "cpu_baseline": {"value": round(g, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(g, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.parallelism == "ep":
        r = run_ep(args, args.workload, rank, world)
        w = r["w"]
        ms = r["total_ms"] / args.steps
        step_bytes = ep_step_bytes(w)
        line = {
            "metric": METRIC, "value": round(job_throughput(step_bytes, world, ms), 1), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_for(w, world, w.T * w.k, "ep"),
            "total_us": round(ms * 1e3, 2), "bytes_per_step_per_rank": step_bytes,
            "gpu_launches": r["kernels_per_step"] * args.steps * world,
            "clocks": r["clocks"],
            "note": "expert parallelism: rank d hosts experts [d E/N, (d+1) E/N); rows cross NVLink "
                    "to the hosting rank; one step per CUDA graph replay",
        }
        if rank == 0:
            print(json.dumps(line), flush=True)
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
        return
    r = run_gpu(args, args.workload, rank, world, with_e2e=True)
    head = summarize(r, args.steps, world, peak, peak_kind)
    w = r["w"]
    e2e = r["e2e"]
    step_bytes = sum(head["bytes_per_step"].values())
    launches = r["launches_per_step"] * args.steps * world
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": config_for(w, world, r["rows_cap"]),
        **{k: head[k] for k in ("dispatch_us", "combine_us", "total_us", "pct_of_peak",
                                "pct_of_spec_peak", "bytes_per_step", "step_us_spread", "roofline")},
        "e2e": {"value": round(job_throughput(step_bytes, world, e2e["ms"]), 3), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"] * world, "d2h_bytes_per_step": e2e["d2h"] * world,
                "ms_per_step": round(e2e["ms"], 4),
                "copies": ("pinned host buffers; inputs up on one stream, y down on another, two "
                           "device sets, so one step's download overlaps the next step's upload")},
        "kernels_per_step": head["kernels_per_step"],
        "timing": head["timing"],
        "clocks": head["clocks"],
    }
    if per_config:
        line["per_config"] = {}
        for name in per_config:
            rp = run_gpu(args, name, rank, world, with_e2e=False)
            s = summarize(rp, args.steps, world, peak, peak_kind)
            s["config"] = config_for(rp["w"], world, rp["rows_cap"])
            line["per_config"][name] = s
            launches += rp["launches_per_step"] * args.steps * world
        # every timed pass above launched this library's kernels only
    line["gpu_launches"] = launches
    line["gpu_launches_note"] = ("kernel nodes of the captured step graph x K, over the headline "
                                 "and per_config timed passes")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        g, desc = time_oracle(w0)
        line["cpu_baseline"] = {"value": round(g, 4), "unit": "GB/s", "cores": 1,
                                "kind": "oracle", "sample": desc}
        cores = len(os.sched_getaffinity(0))
        g, desc = time_oracle(w0, budget_s=5.0, threads=cores)
        line["cpu_baseline_all_cores"] = {"value": round(g, 4), "unit": "GB/s", "cores": cores,
                                          "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
