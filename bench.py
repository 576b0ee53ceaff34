"""Benchmark of the MoonEP hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload training]
                    [--impl reference] [--no-sweep] [--no-extras]
                    [--only KERNEL]

A step is one pass of the whole hot path over one MoE layer of the workload
(default: the training workload, R=16 simulated ranks, 256 experts, 131,072
tokens): moonep_plan -> moonep_prefetch -> moonep_dispatch -> moonep_combine
-> moonep_reduce_grad (the combine gathers the dispatched rows themselves:
the expert computation is out of scope).  Inputs are resident in HBM when the
timed region starts and are larger than L2, so no flush is needed between
steps.  Every kernel is timed with CUDA events on the launching stream;
`value` is the dispatch+combine algorithmic bytes over their device time,
summed over ranks; `e2e` is the same metric through the same calls with the
router output and hidden states copied in from pinned host memory and the
combined output copied back, inside the timed region.

At one GPU the same line also carries the mid workload's step (`mid`), the
inference workload's fallback rows per seed and their throughput cost
(headroom rows versus remote weights, `inference`), and the skew sweep over
maxvio 0..8 at five router seeds each (`sweep`).  Their router outputs are
drawn in spawned worker processes while the GPU measures the main workload.
--only KERNEL times one kernel alone (profiler captures).

Under torchrun every rank runs its own independent replica of the workload
("replicas only": the path is simulated on one GPU, with no exchange between
GPUs); times are the max over ranks.  --impl reference times the CPU oracle
(single-threaded C) on a bounded sample of the same workload, on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from load_balancing_plan_b200 import inputs  # noqa: E402

METRIC = "dispatch+combine GB/s vs HBM peak; plan µs; rows/s flat across maxvio sweep"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# algorithmic bytes (per launch)
# ---------------------------------------------------------------------------

def alg_bytes(cfg, n_replicas=0, n_rx=0, w_elems=0, g_elems=0):
    """Bytes each step must move at minimum.  T = R*S tokens; n_replicas =
    replica pieces with a slot, n_rx = experts with at least one of them.
    dispatch: read x once, write K rows per token, read ids, write dest.
    combine: read K rows per token, write one, read weights and dest.
    prefetch: read each replicated expert's P*H*I bf16 weights once, write
    them to every used slot.
    reduce_grad: read+write the home gradient of each replicated expert,
    read+zero every replica (fp32).  plan: read the ids.
    combine_backward: read grad_out once and the K expert-output rows of each
    token, write the K grad_y rows and grad_w, read weights and dest.
    dispatch_backward: read the K grad rows of each token, write grad_x, read
    dest."""
    T = cfg["R"] * cfg["S"]
    K, H = cfg["K"], cfg["H"]
    row = 2 * H
    return dict(
        dispatch=T * row + T * K * row + 8 * T * K,
        combine=T * K * row + T * row + 8 * T * K,
        prefetch=2 * w_elems * (n_rx + n_replicas),
        reduce_grad=4 * g_elems * (2 * n_rx + 2 * n_replicas),
        plan=4 * T * K,
        combine_backward=T * row + 2 * T * K * row + 12 * T * K,
        dispatch_backward=T * K * row + T * row + 4 * T * K,
    )


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary
    (profiles/dram_traffic.txt: kernel, workload, bytes, then how the figure
    was obtained), as (bytes, source) or (None, None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                if line.startswith("#") or not line.strip():
                    continue
                parts = line.split(None, 3)
                if len(parts) >= 3 and parts[0] == kernel and parts[1] == workload:
                    src = parts[3].strip() if len(parts) > 3 else "profiles/dram_traffic.txt"
                    return float(parts[2]), src
    except OSError:
        pass
    return None, None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index, period=0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                import torch
                pr = torch.cuda.get_device_properties(device_index)
                bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in _REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_over_ranks(local_ms, local_units, world):
    """Max of the timed-region lengths and sum of the units over ranks (the
    identity with one rank).  Returns (max_ms, total_units)."""
    if world <= 1:
        return float(local_ms), float(local_units)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=dev)
    u = torch.tensor([float(local_units)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

class Runner:
    def __init__(self, wl, maxvio, seed, with_weights=True, plan_flags=0, seed_route=None, with_grads=True,
                 route=None):
        import torch
        from load_balancing_plan_b200 import harness
        self.torch = torch
        self.wl = wl
        self.cfg = wl.cfg()
        t0 = time.time()
        if route is None:
            route = inputs.routing(wl.R, wl.L, wl.S, wl.K, seed if seed_route is None else seed_route,
                                   maxvio=maxvio)
        self.route = route
        self.plan_flags = plan_flags
        self.gen_s = time.time() - t0
        we = wl.w_elems if with_weights else 0
        ge = wl.g_elems if with_weights and with_grads else 0
        self.prob = harness.Problem(self.cfg, w_elems=we, g_elems=ge)
        self.prob.set_routing(self.route.topk_idx, self.route.topk_w)
        self.prob.fill_x(seed)
        self.prob.fill_weights(seed)
        self.prob.fill_g_rep(seed)
        self.stream = torch.cuda.current_stream()
        self.with_weights = with_weights
        self.with_grads = with_weights and with_grads
        torch.cuda.synchronize()

    def set_route(self, route):
        """Next router output on the same buffers (same shapes)."""
        self.route = route
        self.prob.set_routing(route.topk_idx, route.topk_w)
        self.torch.cuda.synchronize()

    def step(self, ev=None):
        p = self.prob
        s = self.stream
        if ev is not None:
            ev[0].record(s)
        p.plan(s, self.plan_flags)
        if ev is not None:
            ev[1].record(s)
        if self.with_weights:
            p.prefetch(s)
        if ev is not None:
            ev[2].record(s)
        p.dispatch(s)
        if ev is not None:
            ev[3].record(s)
        p.combine(None, s)
        if ev is not None:
            ev[4].record(s)
        if self.with_grads:
            p.reduce_grad(s)
        if ev is not None:
            ev[5].record(s)

    def launches_per_step(self):
        if self.cfg["B"] == 0 or not self.with_weights:
            return 3
        return 5 if self.with_grads else 4

    def timed(self, steps, warmup, world=1, graph=True):
        """Times `steps` steps after `warmup` untimed ones.  With graph=True
        the step is captured into a CUDA graph of G steps (timing events
        included) and replayed: the timed region replays it steps/G times
        back to back between two events (no host launch latency can show),
        and a second pass of replays, each read back, gives every kernel's
        duration from the events inside the graph.  Returns (total_ms,
        per-kernel lists, clocks, launch mode)."""
        torch = self.torch
        names = ["plan", "prefetch", "dispatch", "combine", "reduce_grad"]
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        G = 10 if steps % 10 == 0 else 1
        g = None
        keep = self.stream
        if graph:
            try:
                cap = torch.cuda.Stream()
                cap.wait_stream(self.stream)
                evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)] for _ in range(G)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    self.stream = cap
                    for i in range(G):
                        self.step(evs[i])
                self.stream = keep
                torch.cuda.synchronize()
                g.replay()
                torch.cuda.synchronize()
            except Exception as exc:  # capture not available: launch eagerly
                self.stream = keep
                g = None
                print("bench: CUDA graph capture failed (%s); timing eager launches" % exc, file=sys.stderr)
                torch.cuda.synchronize()
        if g is not None:
            barrier(world)
            torch.cuda.synchronize()
            with ClockSampler(torch.cuda.current_device()) as clk:
                start = torch.cuda.Event(enable_timing=True)
                end = torch.cuda.Event(enable_timing=True)
                start.record(self.stream)
                for _ in range(steps // G):
                    g.replay()
                end.record(self.stream)
                torch.cuda.synchronize()
            barrier(world)
            total_ms = start.elapsed_time(end)
            per = {n: [] for n in names}
            for _ in range(steps // G):
                g.replay()
                torch.cuda.synchronize()
                for i in range(G):
                    for j, n in enumerate(names):
                        per[n].append(evs[i][j].elapsed_time(evs[i][j + 1]))
            return total_ms, per, clk.summary(), "cuda_graph_%d_steps" % G
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(torch.cuda.current_device()) as clk:
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            start.record(self.stream)
            for i in range(steps):
                self.step(evs[i])
            end.record(self.stream)
            torch.cuda.synchronize()
        barrier(world)
        total_ms = start.elapsed_time(end)
        per = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)] for j, n in enumerate(names)}
        return total_ms, per, clk.summary(), "eager"

    def backward(self, steps, warmup):
        """The training backward pair on the same plan: combine_backward
        (grad_y and grad_w) and dispatch_backward, each timed alone with CUDA
        events; the output gradient is the hidden states and the expert
        outputs are the dispatched rows (values do not change the work).
        Also times copy_out (zero_copy = false) of the dispatched rows.  The
        gradient buffer doubles as copy_out's target (it is rewritten by each
        combine_backward anyway)."""
        torch = self.torch
        from load_balancing_plan_b200 import moonep as mp
        p, cfg, s = self.prob, self.cfg, self.stream
        T, K, H = p.T, cfg["K"], cfg["H"]
        grad_y = torch.empty_like(p.recv)
        grad_w = torch.empty(T * K, dtype=torch.float32, device=p.recv.device)
        grad_x = torch.empty_like(p.out)
        cb = lambda: mp.moonep_combine_backward(cfg, p.ws, p.x, p.recv, p.dest, p.w, grad_y, grad_w, s)
        db = lambda: mp.moonep_dispatch_backward(cfg, p.ws, p.recv, p.dest, grad_x, s)
        # zero_copy = false: the dispatched rows (T*K of them) copied out
        kept = grad_y
        co = lambda: mp.moonep_copy_out(cfg, p.ws, p.recv, kept, s)
        res = {}
        ab = alg_bytes(cfg)
        for name, fn, nbytes in (("combine_backward", cb, ab["combine_backward"]),
                                 ("dispatch_backward", db, ab["dispatch_backward"]),
                                 ("copy_out", co, 2 * T * K * 2 * H)):
            for _ in range(warmup):
                fn()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(s)
            for _ in range(steps):
                fn()
            b.record(s)
            torch.cuda.synchronize()
            us = a.elapsed_time(b) / steps * 1e3
            res[name] = {"us": round(us, 1), "gbs": round(nbytes / us / 1e3, 1), "algorithmic_bytes": nbytes}
        return res

    def e2e(self, steps, warmup):
        """The same calls with every step's router output and hidden states
        copied in from pinned host memory and its combined output copied back
        to pinned host memory, all inside the timed region.  Steps are
        pipelined: two input and two output buffer sets, host-to-device copies
        on one stream, device-to-host copies on another, the hot path on the
        compute stream, ordered by events (a step's kernels wait for its
        inputs; a buffer is refilled only after the step that used it).
        Returns (ms, h2d bytes, d2h bytes, link ms): the last is a separate
        measurement of the host link alone, after the timed region: the same
        steps' host-to-device and device-to-host copies, the same bytes and
        buffers, the two directions at once, no kernels; it is the bound the
        end-to-end time is compared with."""
        torch = self.torch
        p = self.prob
        T, K = self.prob.T, self.cfg["K"]
        n = T * K
        ids_h = torch.from_numpy(self.route.topk_idx.reshape(-1).copy()).pin_memory()
        w_h = torch.from_numpy(self.route.topk_w.reshape(-1).copy()).pin_memory()
        x_h = p.x.cpu().pin_memory()
        outs_h = [torch.empty_like(p.out, device="cpu").pin_memory() for _ in range(2)]
        dev = p.x.device
        ids_d = [p.ids, torch.empty_like(p.ids)]
        w_d = [p.w, torch.empty_like(p.w)]
        x_d = [p.x, torch.empty_like(p.x)]
        out_d = [p.out, torch.empty_like(p.out)]
        comp = self.stream
        h2d = torch.cuda.Stream(device=dev)
        d2h = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        inputs_ready = [ev(), ev()]
        inputs_free = [ev(), ev()]
        out_ready = [ev(), ev()]
        out_free = [ev(), ev()]
        for e in inputs_free + out_free:
            e.record(comp)

        def run(nsteps):
            for i in range(nsteps):
                b = i & 1
                h2d.wait_event(inputs_free[b])
                with torch.cuda.stream(h2d):
                    ids_d[b][:n].copy_(ids_h, non_blocking=True)
                    w_d[b][:n].copy_(w_h, non_blocking=True)
                    x_d[b].copy_(x_h, non_blocking=True)
                inputs_ready[b].record(h2d)
                comp.wait_event(inputs_ready[b])
                comp.wait_event(out_free[b])
                p.ids, p.w, p.x, p.out = ids_d[b], w_d[b], x_d[b], out_d[b]
                self.step()
                inputs_free[b].record(comp)
                out_ready[b].record(comp)
                d2h.wait_event(out_ready[b])
                with torch.cuda.stream(d2h):
                    outs_h[b].copy_(out_d[b], non_blocking=True)
                out_free[b].record(d2h)

        run(warmup)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(h2d)
        run(steps)
        z.record(d2h)
        torch.cuda.synchronize()
        p.ids, p.w, p.x, p.out = ids_d[0], w_d[0], x_d[0], out_d[0]
        h2d_bytes = ids_h.numel() * 4 + w_h.numel() * 4 + x_h.numel() * 2
        d2h_bytes = outs_h[0].numel() * 2

        # the host link alone: both directions' copies of every step at once
        def link(nsteps):
            for i in range(nsteps):
                b = i & 1
                with torch.cuda.stream(h2d):
                    ids_d[b][:n].copy_(ids_h, non_blocking=True)
                    w_d[b][:n].copy_(w_h, non_blocking=True)
                    x_d[b].copy_(x_h, non_blocking=True)
                with torch.cuda.stream(d2h):
                    outs_h[b].copy_(out_d[b], non_blocking=True)

        link(2)
        torch.cuda.synchronize()
        la = torch.cuda.Event(enable_timing=True)
        lh = torch.cuda.Event(enable_timing=True)
        ld = torch.cuda.Event(enable_timing=True)
        la.record(h2d)
        d2h.wait_event(la)
        link(steps)
        lh.record(h2d)
        ld.record(d2h)
        torch.cuda.synchronize()
        link_ms = max(la.elapsed_time(lh), la.elapsed_time(ld))
        return a.elapsed_time(z), h2d_bytes, d2h_bytes, link_ms


def bind_near_gpu(device_index):
    """Restricts this process to the CPUs next to the GPU's PCIe root (its
    NUMA node, as sysfs lists them), so that the pinned host buffers of the
    e2e measurement are allocated in that node's memory and host<->device
    copies do not cross the inter-socket link.  Returns a description, or None
    if the list is not available (nothing changes then)."""
    try:
        import torch
        pr = torch.cuda.get_device_properties(device_index)
        path = "/sys/bus/pci/devices/%04x:%02x:%02x.0/local_cpulist" % (pr.pci_domain_id, pr.pci_bus_id,
                                                                       pr.pci_device_id)
        with open(path) as f:
            spec = f.read().strip()
        cpus = set()
        for part in spec.split(","):
            if "-" in part:
                a, b = part.split("-")
                cpus.update(range(int(a), int(b) + 1))
            elif part:
                cpus.add(int(part))
        use = cpus & os.sched_getaffinity(0)
        if not use:
            return None
        os.sched_setaffinity(0, use)
        return "%d host cpus local to the GPU (%s)" % (len(use), spec)
    except Exception:
        return None


def _route_job(job):
    """Router output for one (workload name, seed, target maxvio), drawn in a
    worker process."""
    name, seed, mv = job
    wl = inputs.WORKLOADS[name]
    return inputs.routing(wl.R, wl.L, wl.S, wl.K, seed, maxvio=mv)


class RoutePool:
    """Draws router outputs in spawned worker processes (no CUDA state is
    inherited) while the GPU measures.  close() before anything is timed on
    the host."""

    def __init__(self, jobs, workers):
        import multiprocessing as mpc
        self.jobs = list(jobs)
        self.pool = mpc.get_context("spawn").Pool(workers) if self.jobs and workers > 0 else None
        self.res = {j: self.pool.apply_async(_route_job, (j,)) for j in self.jobs} if self.pool else {}

    def get(self, job):
        r = self.res.get(job)
        return r.get() if r is not None else _route_job(job)

    def wait(self):
        for r in self.res.values():
            r.wait()

    def close(self):
        if self.pool is not None:
            self.pool.close()
            self.pool.join()
            self.pool = None


def layer_figures(run, steps, warmup, world, graph, peak):
    """Plans once (checking the status), then times `steps` steps of the
    layer.  Returns the per-kernel figures; device times are the max over
    ranks and work units the sum."""
    from load_balancing_plan_b200 import moonep as mp
    run.step()
    info = mp.moonep_plan_read(run.cfg, run.prob.ws)
    if info["status"] & mp.ST_ERROR_MASK:
        raise RuntimeError("plan failed: status 0x%x" % info["status"])
    tabs = mp.moonep_plan_read(run.cfg, run.prob.ws, tables=True)
    slotted = np.asarray(tabs["rep_slot"]) >= 0                # pieces whose weights are prefetched
    n_slot = int(slotted.sum())
    n_rx = len(set(np.asarray(tabs["rep_expert"])[slotted].tolist()))
    w_el = run.prob.w_elems if run.with_weights else 0
    g_el = run.prob.g_elems if run.with_grads else 0
    ab = alg_bytes(run.cfg, n_slot, n_rx, w_el, g_el)
    total_ms, per, clocks, launch_mode = run.timed(steps, warmup, world, graph=graph)
    mean = {k: float(np.mean(v)) for k, v in per.items()}
    dc_ms = sum(per["dispatch"]) + sum(per["combine"])
    max_dc_ms, dc_bytes = reduce_over_ranks(dc_ms, (ab["dispatch"] + ab["combine"]) * steps, world)
    T, K = run.prob.T, run.cfg["K"]
    max_total_ms, rows = reduce_over_ranks(total_ms, T * K * steps, world)
    value = dc_bytes / (max_dc_ms * 1e-3) / 1e9
    shares = {k: sum(v) for k, v in per.items()}
    dom = max(("dispatch", "combine", "prefetch", "reduce_grad"), key=lambda k: shares[k])
    kernel_gbs = {k: (ab[k] / (mean[k] * 1e-3) / 1e9 if mean[k] > 0 and ab[k] else None)
                  for k in ("dispatch", "combine", "prefetch", "reduce_grad")}
    return dict(info=info, n_rx=n_rx, n_slot=n_slot, ab=ab, mean=mean, per=per, value=value,
                ms_per_step=max_total_ms / steps, rows_per_s=rows / (max_total_ms * 1e-3),
                dom=dom, kernel_gbs=kernel_gbs, clocks=clocks, launch_mode=launch_mode,
                frac=value / world / peak)


def short_figures(f, T, K):
    """The per-layer figures an extra workload reports."""
    info = f["info"]
    return {"value": round(f["value"], 2), "unit": UNIT, "ms_per_step": round(f["ms_per_step"], 4),
            "dispatch_combine_frac_of_peak": round(f["frac"], 4),
            "plan_us": round(f["mean"]["plan"] * 1e3, 2),
            "kernel_us": {k: round(v * 1e3, 2) for k, v in f["mean"].items()},
            "kernel_gbs": {k: (round(v, 1) if v else None) for k, v in f["kernel_gbs"].items()},
            "rows_per_s": round(f["rows_per_s"], 1),
            "plan_info": {"n_replicas": info["n_replicas"], "slotted_replicas": f["n_slot"],
                          "replicated_experts": f["n_rx"], "migrated_rows": info["migrated_rows"],
                          "migrated_frac": round(info["migrated_rows"] / (T * K), 4),
                          "fallback_rows": info["fallback_rows"]}}


def wl_desc(wl, route, extra=""):
    return ("%s: R=%d L=%d (N=%d experts) S=%d K=%d H=%d B=%d C=%d C_max=%d, router bias tuned to maxvio "
            "%.2f (achieved %.3f)%s" % (wl.name, wl.R, wl.L, wl.N, wl.S, wl.K, wl.H, wl.B, wl.C, wl.C_max,
                                         route.target if route.target is not None else -1, route.maxvio, extra))


def run_gpu(args):
    import torch
    rank, local_rank, world = rank_env()
    extras = world == 1 and not args.no_extras
    # router outputs for the extra workloads, drawn while the GPU measures
    jobs = []
    if extras:
        jobs += [("inference", s, inputs.WORKLOADS["inference"].maxvio[0]) for s in args.seeds]
        if not args.no_sweep:
            jobs += [("skew", s, mv) for mv in inputs.WORKLOADS["skew"].maxvio for s in args.seeds]
    pool = RoutePool(jobs, min(args.route_workers, len(jobs)))
    torch.cuda.set_device(local_rank)
    host_cpus = bind_near_gpu(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    wl = inputs.WORKLOADS[args.workload]
    target = wl.maxvio[0] if wl.maxvio else None
    from load_balancing_plan_b200 import moonep as mp
    flags = {"headroom": 0, "remote": mp.PLAN_REMOTE_WEIGHTS, "one_group": mp.PLAN_ONE_GROUP}[args.plan_mode]
    if args.plan_mode == "remote":
        # remote weights place every row below C: no headroom is needed
        import dataclasses
        wl = dataclasses.replace(wl, headroom=0.0)
    elif args.plan_mode == "one_group":
        # receivers locked to one home group leave rows on their home ranks
        import dataclasses
        wl = dataclasses.replace(wl, headroom=max(wl.headroom, 1.0))
    peak, peak_kind = measured_peak()
    # inference (no gradients): plan -> prefetch -> dispatch -> combine
    run = Runner(wl, target, seed=args.seed, plan_flags=flags, seed_route=args.route_seed,
                 with_grads=wl.name != "inference")
    f = layer_figures(run, args.steps, args.warmup, world, not args.eager, peak)
    info, ab, mean, dom = f["info"], f["ab"], f["mean"], f["dom"]
    achieved = ab[dom] / (mean[dom] * 1e-3) / 1e9
    bwd = run.backward(max(10, args.steps // 10), args.warmup)

    # the host-timed part waits until the router workers are done
    pool.wait()
    pool.close()
    # a longer stream of steps amortises the pipeline's fill and drain (one step of
    # copies and one of compute are not overlapped at the ends)
    e2e_steps = max(8, args.steps // 4)
    e2e_ms, h2d, d2h, link_ms = run.e2e(e2e_steps, 3)
    max_e2e_ms, e2e_bytes = reduce_over_ranks(e2e_ms, (ab["dispatch"] + ab["combine"]) * e2e_steps, world)
    max_link_ms, _ = reduce_over_ranks(link_ms, 0, world)
    route_main = run.route
    x_gb, recv_gb = run.prob.x.numel() * 2 / 1e9, run.prob.recv.numel() * 2 / 1e9
    with_grads = run.with_grads
    launches = run.launches_per_step() * args.steps
    del run
    torch.cuda.empty_cache()

    extra = {}
    if extras:
        if args.workload != "mid":
            extra["mid"] = run_mid(args, peak)
        extra["ep_emulated"] = run_ep(args, peak)
        extra["inference"] = run_inference(args, peak, pool)
        if not args.no_sweep:
            extra["sweep"] = run_sweep(args, peak, pool)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(wl, route_main, args.cpu_seconds)

    traffic, traffic_src = recorded_traffic(dom, wl.name)
    out = {
        "metric": METRIC, "value": round(f["value"], 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(f["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl_desc(wl, route_main, ", seed %d" % (args.seed if args.route_seed is None
                                                                          else args.route_seed)),
                   "step": "plan -> prefetch -> dispatch -> combine" + (" -> reduce_grad" if with_grads else ""),
                   "weights_per_expert": "bf16 [%d x %d x %d]" % (wl.P, wl.H, wl.I),
                   "grads_per_expert": "fp32 [%d x %d]" % (wl.H, wl.I),
                   "accumulate": "fp32", "parallelism": "replicas%d" % world,
                   "plan_mode": args.plan_mode, "launch": f["launch_mode"], "host_cpus": host_cpus,
                   "l2": "no flush: inputs larger than L2 (x %.2f GB, recv %.2f GB)" % (x_gb, recv_gb)},
        "plan_us": round(mean["plan"] * 1e3, 2),
        "kernel_us": {k: round(v * 1e3, 2) for k, v in mean.items()},
        "kernel_gbs": {k: (round(v, 1) if v else None) for k, v in f["kernel_gbs"].items()},
        "rows_per_s": round(f["rows_per_s"], 1),
        "dispatch_combine_frac_of_peak": round(f["value"] / world / peak, 4),
        "dispatch_combine_frac_of_8tbs": round(f["value"] / world / 8000.0, 4),
        "plan_info": {"n_replicas": info["n_replicas"], "slotted_replicas": f["n_slot"],
                      "migrated_rows": info["migrated_rows"],
                      "migrated_frac": round(info["migrated_rows"] / (wl.T * wl.K), 4),
                      "fallback_rows": info["fallback_rows"], "replicated_experts": f["n_rx"]},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "algorithmic_bytes": ab[dom], "traffic": traffic, "traffic_source": traffic_src},
        "e2e": {"value": round(e2e_bytes / (max_e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(max_e2e_ms / e2e_steps, 4),
                "host_link_ms_per_step": round(max_link_ms / e2e_steps, 4),
                "frac_of_host_link": round(max_link_ms / max_e2e_ms, 4)},
        "gpu_launches": launches,
        "clocks": f["clocks"],
    }
    out["copy_out"] = bwd.pop("copy_out")
    out["backward"] = bwd
    out.update(extra)
    if cpu is not None:
        out["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_mid(args, peak):
    """The mid workload's whole step (plan -> prefetch -> dispatch -> combine
    -> reduce_grad), seed 0."""
    import torch
    wl = inputs.WORKLOADS["mid"]
    run = Runner(wl, wl.maxvio[0], seed=0)
    f = layer_figures(run, args.extra_steps, 3, 1, not args.eager, peak)
    out = {"workload": wl_desc(wl, run.route, ", seed 0"),
           "step": "plan -> prefetch -> dispatch -> combine -> reduce_grad", **short_figures(f, wl.T, wl.K)}
    del run
    torch.cuda.empty_cache()
    return out


def run_ep(args, peak, workload="mid"):
    """A workload's step (mid by default) through the expert-parallel calls,
    its R ranks emulated on this GPU (each rank's own buffers, peers through
    peer-pointer tables; each rank's counting launch stores its counts into
    every rank's counts_all): per rank count -> plan -> prefetch -> dispatch
    -> combine -> combine_backward -> dispatch_backward -> reduce_grad, rank
    after rank for each call.  Every kernel is launched once per rank;
    the figures are the sums over the ranks' launches (CUDA events around
    each phase on the launching stream).  One GPU per rank is not measured
    here."""
    import torch
    from load_balancing_plan_b200 import ep
    wl = inputs.WORKLOADS[workload]
    cfg = wl.cfg()
    route = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, maxvio=wl.maxvio[0])
    em = ep.Emulation(cfg, w_elems=wl.w_elems, g_elems=wl.g_elems)
    em.set_routing(route.topk_idx, route.topk_w)
    for q, rb in enumerate(em.ranks):
        inputs.cb_fill_torch(rb.x.view(torch.bfloat16), 0, inputs.STREAM_X, offset=q * wl.S * wl.H)
        inputs.cb_fill_torch(rb.w_home.view(torch.bfloat16), 0, inputs.STREAM_W, offset=q * wl.L * wl.w_elems)
        inputs.cb_fill_torch(rb.g_home, 0, inputs.STREAM_G_HOME, offset=q * wl.L * wl.g_elems)
    s = torch.cuda.current_stream()
    # the backward pair: each rank's combine output stands in for its
    # grad_out; grad_y lands on the ranks that hold the rows
    dev = em.ranks[0].recv.device
    grad_y = [torch.empty_like(rb.recv) for rb in em.ranks]
    grad_y_peers = ep.peer_table(grad_y, dev)
    grad_w = [torch.empty_like(rb.w) for rb in em.ranks]
    grad_x = [torch.empty_like(rb.x) for rb in em.ranks]
    grad_out = [rb.out for rb in em.ranks]
    phases = [("plan", lambda: em.plan(exchange=True)), ("prefetch", em.prefetch), ("dispatch", em.dispatch),
              ("combine", em.combine),
              ("combine_backward", lambda: em.combine_backward(grad_out, grad_y_peers, grad_w)),
              ("dispatch_backward", lambda: em.dispatch_backward(grad_y_peers, grad_x)),
              ("reduce_grad", em.reduce_grad)]
    for _ in range(3):
        for _, fn in phases:
            fn()
    torch.cuda.synchronize()
    info = em.ranks[0].read_plan(tables=True)
    if info["status"] & 0xFF:
        raise RuntimeError("expert-parallel plan failed: status 0x%x" % info["status"])
    n_rx = len(set(np.asarray(info["rep_expert"]).tolist()))
    ab = alg_bytes(cfg, info["n_replicas"], n_rx, wl.w_elems, wl.g_elems)
    # one rank per GPU: every receiver reads its experts' weights from the
    # home rank itself, one read and one write per slot
    ab["prefetch"] = 2 * 2 * wl.w_elems * info["n_replicas"]
    steps = args.extra_steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)] for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(s)
        for j, (_, fn) in enumerate(phases):
            fn()
            ev[i][j + 1].record(s)
    torch.cuda.synchronize()
    us = {name: float(np.mean([ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps)])) * 1e3
          for j, (name, _) in enumerate(phases)}
    total_ms = float(np.mean([ev[i][0].elapsed_time(ev[i][-1]) for i in range(steps)]))
    dc = ab["dispatch"] + ab["combine"]
    value = dc / ((us["dispatch"] + us["combine"]) * 1e-6) / 1e9
    out = {"workload": wl_desc(wl, route, ", seed 0; %d ranks emulated on one GPU" % wl.R),
           "step": "per rank: count with the counts' exchange (moonep_ep_count_exchange) -> plan -> prefetch -> "
                   "dispatch -> combine -> combine_backward -> dispatch_backward -> reduce_grad",
           "value": round(value, 2), "unit": UNIT, "dispatch_combine_frac_of_peak": round(value / peak, 4),
           "ms_per_step": round(total_ms, 4), "launch": "eager, one launch per rank and call",
           "phase_us": {k: round(v, 2) for k, v in us.items()},
           "phase_gbs": {k: (round(ab[k] / (v * 1e-6) / 1e9, 1) if ab[k] and k != "plan" else None)
                         for k, v in us.items()}}
    del em, grad_y, grad_w, grad_x, grad_out
    torch.cuda.empty_cache()
    return out


def run_inference(args, peak, pool):
    """The inference workload (B = 4 slots, C_max = 1.25 C): headroom-rule
    fallback rows for every seed, then the step (plan -> prefetch -> dispatch
    -> combine) timed on the seed with the most fallback rows under the
    headroom rule and under remote weights (the pages' inference fallback),
    on the same buffers: the difference is the fallback's throughput cost."""
    import torch
    from load_balancing_plan_b200 import moonep as mp
    wl = inputs.WORKLOADS["inference"]
    mv = wl.maxvio[0]
    routes = {s: pool.get(("inference", s, mv)) for s in args.seeds}
    run = Runner(wl, mv, seed=0, with_grads=False, route=routes[args.seeds[0]])
    per_seed = {}
    for s in args.seeds:
        run.set_route(routes[s])
        run.prob.plan()
        info = mp.moonep_plan_read(run.cfg, run.prob.ws)
        per_seed[str(s)] = {"maxvio": round(routes[s].maxvio, 3), "fallback_rows": info["fallback_rows"],
                            "n_replicas": info["n_replicas"], "migrated_rows": info["migrated_rows"]}
    worst = max(args.seeds, key=lambda s: (per_seed[str(s)]["fallback_rows"], -s))
    run.set_route(routes[worst])
    modes = {}
    for mode, fl in (("headroom", 0), ("remote", mp.PLAN_REMOTE_WEIGHTS)):
        run.plan_flags = fl
        f = layer_figures(run, args.extra_steps, 3, 1, not args.eager, peak)
        modes[mode] = short_figures(f, wl.T, wl.K)
    hm, rm = modes["headroom"], modes["remote"]
    out = {"workload": wl_desc(wl, routes[worst]), "step": "plan -> prefetch -> dispatch -> combine",
           "fallback_rows_per_seed": per_seed, "timed_seed": worst,
           "fallback_rows": hm["plan_info"]["fallback_rows"],
           "fallback_cost": {"ms_per_step_headroom": hm["ms_per_step"], "ms_per_step_remote": rm["ms_per_step"],
                             "step_time_ratio": round(hm["ms_per_step"] / rm["ms_per_step"], 4),
                             "dispatch_combine_gbs_headroom": hm["value"],
                             "dispatch_combine_gbs_remote": rm["value"]},
           "headroom": hm, "remote": rm}
    del run
    torch.cuda.empty_cache()
    return out


def run_sweep(args, peak, pool):
    """plan -> dispatch -> combine on the skew-sweep workload at each target
    maxvio and seed: rows/s should not move with the skew.  One set of
    buffers serves every point (only the router output changes)."""
    import torch
    from load_balancing_plan_b200 import moonep as mp
    wl = inputs.WORKLOADS["skew"]
    ab = alg_bytes(wl.cfg())
    run = None
    points = {}
    all_rps = []
    for mv in wl.maxvio:
        seeds = {}
        for s in args.seeds:
            route = pool.get(("skew", s, mv))
            if run is None:
                run = Runner(wl, mv, seed=0, with_weights=False, route=route)
            else:
                run.set_route(route)
            total_ms, per, _, _ = run.timed(args.sweep_steps, 3, graph=not args.eager)
            info = mp.moonep_plan_read(run.cfg, run.prob.ws)
            if info["status"] & mp.ST_ERROR_MASK:
                raise RuntimeError("sweep plan failed: status 0x%x" % info["status"])
            d = float(np.mean(per["dispatch"]))
            c = float(np.mean(per["combine"]))
            rps = run.prob.T * wl.K / (total_ms / args.sweep_steps * 1e-3)
            all_rps.append(rps)
            seeds[str(s)] = {
                "maxvio": round(route.maxvio, 3),
                "plan_us": round(float(np.mean(per["plan"])) * 1e3, 2),
                "dispatch_gbs": round(ab["dispatch"] / (d * 1e-3) / 1e9, 1),
                "combine_gbs": round(ab["combine"] / (c * 1e-3) / 1e9, 1),
                "dispatch_combine_frac": round((ab["dispatch"] + ab["combine"]) / ((d + c) * 1e-3) / 1e9 / peak, 4),
                "rows_per_s": round(rps, 1),
                "migrated_frac": round(info["migrated_rows"] / (run.prob.T * wl.K), 4),
                "n_replicas": info["n_replicas"], "fallback_rows": info["fallback_rows"],
            }
        rp = [v["rows_per_s"] for v in seeds.values()]
        points["%g" % mv] = {"seeds": seeds, "rows_per_s_mean": round(float(np.mean(rp)), 1),
                             "rows_per_s_spread_over_seeds": round(max(rp) / min(rp) - 1.0, 4),
                             "plan_us_mean": round(float(np.mean([v["plan_us"] for v in seeds.values()])), 2),
                             "migrated_frac_mean": round(float(np.mean([v["migrated_frac"]
                                                                        for v in seeds.values()])), 4)}
    del run
    torch.cuda.empty_cache()
    means = [v["rows_per_s_mean"] for v in points.values()]
    return {"workload": "skew: R=8 L=32 S=8192 K=8 H=7168 B=32, seeds %s, step = plan -> dispatch -> combine"
                        % ",".join(str(s) for s in args.seeds),
            "points": points, "rows_per_s_spread": round(max(all_rps) / min(all_rps) - 1.0, 4),
            "rows_per_s_spread_of_means": round(max(means) / min(means) - 1.0, 4)}


# ---------------------------------------------------------------------------
# the CPU oracle arm (reference / cpu_baseline)
# ---------------------------------------------------------------------------

class OracleArm:
    """The oracle (as it stands, single-threaded C) on a bounded sample of the
    workload: one step is the plan over all T*K ids, then dispatch and
    combine over the first n tokens (n calibrated once to a time budget)."""

    def __init__(self, wl, route):
        import oracle
        oracle.build()
        self.oracle = oracle
        self.wl, self.route, self.cfg = wl, route, wl.cfg()
        # host receive buffer: only the rows the sample touches get committed
        self.recv = np.empty((wl.R * self.cfg["C_max"], wl.H), np.uint16)
        self.x = None

    def _inputs(self, n):
        if self.x is None or self.x.shape[0] < n:
            self.x = inputs.cb_bf16_np(0, inputs.STREAM_X, np.arange(n * self.wl.H)).reshape(n, self.wl.H)

    def step(self, n):
        o, wl = self.oracle, self.wl
        T, K = wl.T, wl.K
        self._inputs(n)
        t0 = time.perf_counter()
        pl = o.plan(self.cfg, self.route.topk_idx)
        t1 = time.perf_counter()
        d = np.ascontiguousarray(pl["dest"].reshape(T, K)[:n])
        w = np.ascontiguousarray(self.route.topk_w.reshape(T, K)[:n])
        t2 = time.perf_counter()
        o.dispatch(self.cfg, d, self.x[:n], self.recv, n_tokens=n)
        o.combine(self.cfg, d, self.recv, w, n_tokens=n)
        t3 = time.perf_counter()
        b = alg_bytes(dict(self.cfg, S=1, R=n))   # bytes of n tokens
        return {"gbs": (b["dispatch"] + b["combine"]) / (t3 - t2) / 1e9, "plan_us": (t1 - t0) * 1e6,
                "rows_per_s": n * K / (t3 - t2), "tokens": n, "seconds": (t1 - t0) + (t3 - t2)}

    def calibrate(self, seconds):
        """Tokens per step so that a step takes about `seconds`: a first
        small step touches the host buffers (its page faults would inflate
        the estimate), a second, larger one is timed."""
        self.step(min(self.wl.T, 128))
        n = min(self.wl.T, 1024)
        r = self.step(n)
        per_tok = max(r["seconds"] - r["plan_us"] * 1e-6, 1e-7) / n
        return int(max(1, min(self.wl.T, (seconds - r["plan_us"] * 1e-6) / per_tok)))


def host_cpu():
    """The host CPU's model name and the CPUs this process may use."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": len(os.sched_getaffinity(0))}


class one_core:
    """Pins the process to one of its CPUs for the duration (the oracle is
    single-threaded C; this keeps it on one core), then restores the set."""

    def __enter__(self):
        self.saved = os.sched_getaffinity(0)
        self.core = min(self.saved)
        os.sched_setaffinity(0, {self.core})
        return self

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.saved)
        return False


def cpu_baseline(wl, route, seconds):
    info = host_cpu()
    arm = OracleArm(wl, route)
    with one_core():
        n = arm.calibrate(seconds)
        r = arm.step(n)
    return {"value": round(r["gbs"], 4), "unit": UNIT, "cores": 1, "kind": "oracle", **info,
            "plan_us": round(r["plan_us"], 1), "rows_per_s": round(r["rows_per_s"], 1),
            "sample": "oracle plan over all %d ids, then dispatch+combine over the first %d of %d "
                      "tokens (%.1f s, single-threaded C)" % (wl.T * wl.K, r["tokens"], wl.T, r["seconds"])}


def run_reference(args):
    rank, _, world = rank_env()
    if rank != 0:
        return
    wl = inputs.WORKLOADS[args.workload]
    target = wl.maxvio[0] if wl.maxvio else None
    route = inputs.routing(wl.R, wl.L, wl.S, wl.K, args.seed, maxvio=target)
    arm = OracleArm(wl, route)
    info = host_cpu()
    with one_core():
        n = arm.calibrate(args.cpu_seconds * 6.0 / max(1, args.steps + args.warmup))
        for _ in range(args.warmup):
            arm.step(n)
        res = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            res.append(arm.step(n))
        wall = time.perf_counter() - t0
    gbs = float(np.mean([r["gbs"] for r in res]))
    out = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "%s: R=%d L=%d S=%d K=%d H=%d B=%d, maxvio %.2f"
                               % (wl.name, wl.R, wl.L, wl.S, wl.K, wl.H, wl.B, route.maxvio),
                   "accumulate": "fp32", "parallelism": "cpu"},
        "plan_us": round(float(np.mean([r["plan_us"] for r in res])), 1),
        "rows_per_s": round(float(np.mean([r["rows_per_s"] for r in res])), 1),
        "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle", **info,
                         "sample": "per step: oracle plan over all %d ids, dispatch+combine over the "
                                   "first %d tokens" % (wl.T * wl.K, n)},
        "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


KERNELS = ("plan", "prefetch", "dispatch", "combine", "reduce_grad", "combine_backward", "dispatch_backward")


class PlanOnly:
    """The buffers of the plan alone: it reads the ids and writes only the
    workspace."""

    def __init__(self, cfg, route):
        import torch
        from load_balancing_plan_b200 import moonep as mp
        self.cfg, self.mp = cfg, mp
        self.ids = torch.from_numpy(np.ascontiguousarray(route.topk_idx.reshape(-1))).cuda()
        self.ws = torch.zeros(mp.moonep_plan_workspace_bytes(cfg) // 4, dtype=torch.int32, device="cuda")
        self.w_elems = self.g_elems = 0
        self.prefetch = self.dispatch = self.combine = self.reduce_grad = None

    def plan(self):
        self.mp.moonep_plan(self.cfg, self.ids, self.ws)


def run_only(args):
    """One kernel of the step alone, for profiler captures and kernel-alone
    timings: the buffers that kernel needs (weights only for prefetch,
    gradients only for reduce_grad), one plan (and a dispatch before combine),
    then `warmup` untimed and `steps` timed launches of that kernel, each
    bracketed by CUDA events on the launching stream.  Prints one JSON line
    with the median launch time and the algorithmic GB/s."""
    import torch
    from load_balancing_plan_b200 import harness, moonep as mp
    torch.cuda.set_device(0)
    wl = inputs.WORKLOADS[args.workload]
    route = inputs.routing(wl.R, wl.L, wl.S, wl.K, args.seed, maxvio=wl.maxvio[0] if wl.maxvio else None,
                           alpha=wl.alpha)
    cfg = wl.cfg()
    k = args.only
    if k == "plan":
        prob = PlanOnly(cfg, route)
    else:
        prob = harness.Problem(cfg, w_elems=wl.w_elems if k == "prefetch" else 0,
                               g_elems=wl.g_elems if k == "reduce_grad" else 0)
        prob.set_routing(route.topk_idx, route.topk_w)
        prob.fill_x(args.seed)
        prob.fill_weights(args.seed)
        prob.fill_g_rep(args.seed)
    prob.plan()
    pre = 0
    if k in ("combine", "combine_backward", "dispatch_backward"):
        prob.dispatch()
        pre = 1
    if k in ("combine_backward", "dispatch_backward"):
        # the training backward pair on the dispatched rows: grad_out = x,
        # the expert outputs = the dispatched rows
        grad_y = torch.empty_like(prob.recv)
        grad_w = torch.empty(prob.T * cfg["K"], dtype=torch.float32, device=prob.recv.device)
        grad_x = torch.empty_like(prob.out)
    torch.cuda.synchronize()
    info = mp.moonep_plan_read(cfg, prob.ws)
    if info["status"] & mp.ST_ERROR_MASK:
        raise RuntimeError("plan failed: status 0x%x" % info["status"])
    tabs = mp.moonep_plan_read(cfg, prob.ws, tables=True)
    slotted = np.asarray(tabs["rep_slot"]) >= 0
    n_slot = int(slotted.sum())
    n_rx = len(set(np.asarray(tabs["rep_expert"])[slotted].tolist()))
    ab = alg_bytes(cfg, n_slot, n_rx, prob.w_elems, prob.g_elems)[k]
    s = torch.cuda.current_stream()
    if k == "combine_backward":
        fn = lambda: mp.moonep_combine_backward(cfg, prob.ws, prob.x, prob.recv, prob.dest, prob.w, grad_y, grad_w, s)
    elif k == "dispatch_backward":
        fn = lambda: mp.moonep_dispatch_backward(cfg, prob.ws, prob.recv, prob.dest, grad_x, s)
    else:
        fn = {"plan": prob.plan, "prefetch": prob.prefetch, "dispatch": prob.dispatch,
              "combine": prob.combine, "reduce_grad": prob.reduce_grad}[k]
    for _ in range(args.warmup):
        fn()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    for i in range(args.steps):
        ev[2 * i].record(s)
        fn()
        ev[2 * i + 1].record(s)
    torch.cuda.synchronize()
    us = float(np.median([ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)])) * 1e3
    info = mp.moonep_plan_read(cfg, prob.ws)
    if info["status"] & mp.ST_ERROR_MASK:
        raise RuntimeError("%s failed: status 0x%x" % (k, info["status"]))
    peak, peak_kind = measured_peak()
    print(json.dumps({"kernel": k, "workload": wl_desc(wl, route, ", seed %d" % args.seed),
                      "launches": args.warmup + args.steps + 1 + pre, "us": round(us, 2),
                      "algorithmic_bytes": ab, "gbs": round(ab / us / 1e3, 1),
                      "frac_of_peak": round(ab / us / 1e3 / peak, 4), "peak_kind": peak_kind,
                      "n_replicas": info["n_replicas"], "replicated_experts": n_rx}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="training", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--route-seed", type=int, default=None,
                    help="seed of the router output (default: --seed)")
    ap.add_argument("--plan-mode", default="headroom", choices=["headroom", "remote", "one_group"],
                    help="overflow beyond a receiver's slots: headroom rows on the home rank, or remote "
                         "weights; one_group: receivers take replicas of one home group only")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--only", choices=KERNELS + ("ep",), default=None,
                    help="time one kernel alone on the workload (profiler captures); ep: the workload's "
                         "expert-parallel step, its ranks emulated on this GPU")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the main workload (no mid, inference or sweep figures)")
    ap.add_argument("--seeds", type=lambda v: [int(x) for x in v.split(",")], default=[0, 1, 2, 3, 4],
                    help="router seeds of the sweep and the inference fallback count")
    ap.add_argument("--extra-steps", type=int, default=20, help="timed steps of each extra workload")
    ap.add_argument("--route-workers", type=int, default=6,
                    help="worker processes drawing the extra workloads' router outputs")
    ap.add_argument("--eager", action="store_true", help="launch every step from the host (no CUDA graph)")
    ap.add_argument("--sweep-steps", type=int, default=20)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU oracle sample budget (the reference arm uses 6x this over all its steps)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.only == "ep":
        # the expert-parallel step alone (ranks emulated on this GPU), for
        # profiler captures: 3 untimed steps, then --steps timed ones
        import torch
        torch.cuda.set_device(0)
        peak, _ = measured_peak()
        args.extra_steps = args.steps
        print(json.dumps(dict(run_ep(args, peak, args.workload), kernel="ep")), flush=True)
    elif args.only:
        run_only(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
