#!/usr/bin/env python
"""SinkRouter decode-attention benchmark on B200.

One step = one routed decode step of one attention layer (sr_route then
sr_decode_attention, through the C ABI) on synthetic inputs shaped like the
Llama-3.1-8B 128K-context decode layer: batch 1, 32 query / 8 KV heads,
head_dim 128, bf16 cache, 4 of 8 KV groups planted sinks, tau 0.6.

Timing: K layer-steps back to back in one CUDA graph, rotating over input sets
that together exceed L2, one event pair around all of them; the graph is
replayed once untimed, then once timed.

Prints one JSON line (rank 0): µs per layer-step (lower is better), effective
HBM GB/s over the bytes the step must move, the roofline of the decode kernel
against the HBM copy bandwidth (measured, else the fallback), the same kernel
with routing disabled (tau = +inf), the fused single launch, the per-step
protocol (flush, events) for comparison, the append step (RoPE + KV append +
routing, then the scan), the 512K sink-fraction sweep, short contexts and the
other workloads (one GPU), the fp64 CPU oracle on this host's cores, end-to-end
figures with host buffers (every input each step; and the serving view, only
the new token's projections), and the SM clocks seen during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --multilayer        # per-token latency of a gated 32-layer graph
    python bench.py --proxy-quality     # routing proxy vs full-attention sink event
    python bench.py --context-parallel  # one 512K layer-step sharded over the ranks

Multi-GPU (torchrun): every rank runs its own independent layer-step (the
units of a decode step share nothing); time is the max over ranks and the value
is that time divided by all layer-steps of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention µs/layer-step and effective HBM GB/s (% of peak) at 128K/512K ctx"
UNIT = "us/layer-step"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the copy bandwidth above is the roofline)
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_kernel_llama8b_128k.md")
DECODE_SOURCE = os.path.join(ROOT, "kv_cache_routing_sr_b200", "csrc", "sr_decode.cu")
L2_FLUSH_BYTES = 256 << 20

NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="llama8b_128k")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--no-sweep", action="store_true", help="skip the 512K sink-fraction sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--context-parallel", action="store_true",
                    help="instead of the contract line: one 512K layer-step (half the groups sinks) sharded over "
                         "the --gpus ranks by position: partial scans, one all-gather, the combine (strong scaling)")
    ap.add_argument("--multilayer", action="store_true",
                    help="instead of the contract line: per-token attention latency of a 32-layer stack, "
                         "CUDA-graph captured, at 128K/256K/512K context, routed vs routing disabled")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--profile", metavar="WORKLOAD", default=None,
                    help="instead of the contract line: run --warmup + --steps eager two-call steps of one workload "
                         "(optionally at --max-ctx) and print a one-line summary; the command the ncu captures in "
                         "profiles/ run")
    ap.add_argument("--max-ctx", type=int, default=None, help="context of the --profile workload")
    ap.add_argument("--proxy-quality", action="store_true",
                    help="instead of the contract line: precision / recall / F1 of the cosine routing proxy "
                         "against the full-attention position-0 weight, on graded synthetic inputs")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


# ---------------------------------------------------------------------------------------
# helpers shared by both arms

def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            v = json.load(f).get("hbm_gbs")
        if v:
            return float(v), "measured"
    except (OSError, ValueError):
        pass
    return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic():
    """dram bytes per launch of the decode kernel from the committed ncu summary,
    valid only while the kernel source still has the hash it was captured at."""
    try:
        text = open(PROFILE_SUMMARY).read()
        src = hashlib.sha256(open(DECODE_SOURCE, "rb").read()).hexdigest()
    except OSError:
        return None
    m_t = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    m_h = re.search(r"^decode_source_sha256:\s*([0-9a-f]+)", text, re.M)
    if not m_t or not m_h or m_h.group(1) != src:
        return None
    return float(m_t.group(1))


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device, world: int) -> float:
    """Max of a per-rank float over all ranks (identity with one rank). The
    device is the process group's: a CUDA device for NCCL, the CPU for gloo."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_us(max_total_ms: float, steps: int, world: int) -> tuple[float, float]:
    """(slowest rank's µs per layer-step, whole-job µs per layer-step): every rank
    runs `steps` independent layer-steps, so the job completes world*steps of
    them in the slowest rank's time."""
    per_rank = max_total_ms * 1e3 / steps
    return per_rank, per_rank / world


def active_units_of(active_list_cpu):
    n = int(active_list_cpu[0])
    return [int(u) for u in active_list_cpu[1:1 + n]]


def describe_config(x, n_active, n_gpus):
    return {
        "workload": x.workload.name,
        "description": x.workload.description,
        "batch": x.batch, "context": x.max_seq_len, "q_heads": x.n_q_heads, "kv_heads": x.n_kv_heads,
        "head_dim": 128, "tau": x.tau, "units": x.batch * x.n_kv_heads, "active_units": n_active,
        "seq_lens": [int(v) for v in x.seq_lens.cpu().tolist()][:8],
        "l2": f"inputs larger than L2: the steps rotate over {n_input_sets(x)} independently seeded input sets "
              f"({n_input_sets(x) * x.k_cache.numel() * 4 / 2**30:.2f} GiB of K/V), no flush",
        "parallelism": f"replicas x{n_gpus} (independent layer-steps, no collective on the data path)",
    }


# ---------------------------------------------------------------------------------------
# clock sampling (NVML reads only)

class ClockSampler:
    def __init__(self, torch_device_index: int, period_s: float = 0.01):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            h = None
            try:
                bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self.h))

    def _loop(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                self.samples.append((mhz, self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if not self.ok:
            return
        self.samples = []
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()

    def stop(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        self._stop.set()
        self._t.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [name for b, name in NVML_REASONS.items() if bits & b]
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# our arm

def _captured_steps(native, dec, x, tau, steps, flush, split_events, fused, rotate=None):
    """Capture `steps` layer-steps in ONE CUDA graph, as a decode forward would
    run them: before each step an L2 flush (a 256 MiB read), then an event and
    the step, then an event. The step is either the single fused launch
    (sr_route_decode_attention) or sr_route then sr_decode_attention; for the
    latter, split_events=True puts an event between the two kernels (per-kernel
    times), otherwise the decode launch overlaps routing through its
    programmatic dependency."""
    import torch
    # external events: recorded as timestamps by the graph's event nodes
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
    xs = rotate or [x]
    side = torch.cuda.Stream(device=x.q.device)
    side.wait_stream(torch.cuda.current_stream(x.q.device))
    with torch.cuda.stream(side):  # warm-up outside the capture
        for xi in xs:
            dec.step(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, tau)
            dec.step_fused(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, tau)
        if flush is not None:
            flush.sum()
    torch.cuda.current_stream(x.q.device).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        for i in range(steps):
            xi = xs[i % len(xs)]
            args = (xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens)
            if flush is not None:
                flush.sum()
            ev[i][0].record(st)
            if fused:
                native.route_decode_attention(*args, tau, dec.out, dec.route_mask, dec.active_list, 0,
                                              dec.workspace)
            else:
                native.route(xi.q, xi.k0, tau, dec.route_mask, dec.active_list)
                if split_events:
                    ev[i][1].record(st)
                native.decode_attention(*args, dec.active_list, dec.out, 0, dec.workspace)
            ev[i][2].record(st)
    g.sr_events = ev  # recorded on every replay: they must live as long as the graph
    return g, ev


def time_steps(native, dec, x, tau, steps, warmup, flush, barrier, fused, rotate=None):
    """Per-step device times (ms): events bracket the step only. flush=None
    skips the L2 flush; `rotate` cycles the steps over several input sets."""
    import torch
    gw, _ = _captured_steps(native, dec, x, tau, warmup, flush, False, fused, rotate)
    g, ev = _captured_steps(native, dec, x, tau, steps, flush, False, fused, rotate)
    gw.replay()
    g.replay()  # untimed: a graph's first replay pays its one-time launch set-up
    barrier()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    barrier()
    return [e[0].elapsed_time(e[2]) for e in ev]


def time_back_to_back(native, dec, xs, tau, steps, warmup, fused=False, barrier=lambda: None):
    """K layer-steps back to back in one CUDA graph, cycling over the input sets
    `xs` (together larger than L2, so no flush is needed), timed as a block by
    one event pair: (total ms, steps). This is how a decode forward runs its
    layers; each step's launch overlaps the previous step's tail through the
    programmatic dependency."""
    import torch
    dev = xs[0].q.device
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for xi in xs:
            dec.step(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, tau)
            dec.step_fused(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, tau)
    torch.cuda.current_stream(dev).wait_stream(side)

    def capture(n):
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            st = torch.cuda.current_stream()
            e0.record(st)
            for i in range(n):
                xi = xs[i % len(xs)]
                args = (xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens)
                if fused:
                    native.route_decode_attention(*args, tau, dec.out, dec.route_mask, dec.active_list, 0,
                                                  dec.workspace)
                else:
                    native.route(xi.q, xi.k0, tau, dec.route_mask, dec.active_list)
                    native.decode_attention(*args, dec.active_list, dec.out, 0, dec.workspace)
            e1.record(st)
        # the graph records these events on every replay: they must live as
        # long as the graph
        g.sr_events = (e0, e1)
        return g, e0, e1

    g, e0, e1 = capture(steps)
    # warm-up: one untimed replay of the same K steps (at least `warmup`); the
    # first replay of a graph also pays its one-time launch set-up (tens of us
    # before its first kernel starts), which is not part of any step
    for _ in range(max(1, -(-warmup // steps))):
        g.replay()
    barrier()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1), steps


def time_kernels(native, dec, x, tau, steps, flush, rotate=None):
    """Per-kernel device times (ms) of the two-call step with an event between
    the two kernels (which also removes their overlap). flush=None skips the L2
    flush; `rotate` cycles the steps over several input sets."""
    import torch
    g, ev = _captured_steps(native, dec, x, tau, steps, flush, True, False, rotate=rotate)
    g.replay()  # untimed: a graph's first replay pays its one-time launch set-up
    g.replay()
    torch.cuda.synchronize()
    return [e[0].elapsed_time(e[1]) for e in ev], [e[1].elapsed_time(e[2]) for e in ev]


class AppendInputs:
    """Inputs of the decode step that starts from the un-rotated projections
    (sr_rope_append_route then sr_decode_attention) on workload x: every
    sequence's last cache slot takes the new token, so after the append the
    scan covers the workload's full context. q_in is the workload's planted
    query rotated back to that slot (by the library's own kernel, with the sine
    table negated), so routing sees the same groups as the two-call step.
    Each timed step restores seq_lens from seq_saved before its start event."""

    def __init__(self, native, inputs, x):
        import torch
        dev = x.q.device
        B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
        self.seq_saved = (x.seq_lens - 1).clone()
        self.seq_lens = self.seq_saved.clone()
        self.cos, self.sin = inputs.rope_tables(x.max_seq_len, device=dev)
        _, self.k_new, self.v_new = inputs.make_projections(B, Hq, Hkv, seed=x.seed + 17, device=dev)
        # rotate the planted query back: one call per distinct slot, on
        # one-slot scratch caches, with a one-row table (row p, sines negated)
        self.q_in = torch.empty_like(x.q)
        z1 = torch.zeros((1, Hkv, 1, 128), dtype=torch.bfloat16, device=dev)
        for b, p in enumerate(self.seq_saved.tolist()):
            zr = torch.zeros((1, Hkv, 128), dtype=torch.bfloat16, device=dev)
            native.rope_append_route(x.q[b:b + 1].contiguous(), zr, zr.clone(), self.cos[p:p + 1].contiguous(),
                                     (-self.sin[p:p + 1]).contiguous(), torch.zeros(1, dtype=torch.int32, device=dev),
                                     z1.clone(), z1.clone(), zr.clone(), zr.clone(), float("inf"),
                                     q_out=self.q_in[b:b + 1])
        torch.cuda.synchronize()

    def step(self, native, dec, x, tau):
        self.seq_lens.copy_(self.seq_saved)
        return dec.append_step(self.q_in, self.k_new, self.v_new, self.cos, self.sin, x.k_cache, x.v_cache, x.k0,
                               x.v0, self.seq_lens, tau)


class AppendSequence:
    """Inputs of `visits` consecutive append steps on workload x: visit t puts
    the new token of every sequence at slot L - visits + t, so the last visit's
    scan covers the full context; each visit's un-rotated query is the planted
    query rotated back to its slot (by the library's own kernel), so routing
    sees the same groups at every visit. reset() restores the lengths before a
    graph replay."""

    def __init__(self, native, inputs, x, visits):
        import torch
        dev = x.q.device
        B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
        self.seq_saved = (x.seq_lens - visits).clone()
        self.seq_lens = self.seq_saved.clone()
        self.cos, self.sin = inputs.rope_tables(x.max_seq_len, device=dev)
        _, self.k_new, self.v_new = inputs.make_projections(B, Hq, Hkv, seed=x.seed + 17, device=dev)
        z1 = torch.zeros((1, Hkv, 1, 128), dtype=torch.bfloat16, device=dev)
        self.q_in = []
        for t in range(visits):
            q_in = torch.empty_like(x.q)
            for b, p0 in enumerate(self.seq_saved.tolist()):
                p = p0 + t
                zr = torch.zeros((1, Hkv, 128), dtype=torch.bfloat16, device=dev)
                native.rope_append_route(x.q[b:b + 1].contiguous(), zr, zr.clone(), self.cos[p:p + 1].contiguous(),
                                         (-self.sin[p:p + 1]).contiguous(),
                                         torch.zeros(1, dtype=torch.int32, device=dev), z1.clone(), z1.clone(),
                                         zr.clone(), zr.clone(), float("inf"), q_out=q_in[b:b + 1])
            self.q_in.append(q_in)
        torch.cuda.synchronize()

    def reset(self):
        self.seq_lens.copy_(self.seq_saved)


def time_append_back_to_back(native, dec, xs, seqs, tau, steps, warmup):
    """K append steps (sr_rope_append_route, sr_decode_attention) back to back
    in one CUDA graph, cycling over the input sets `xs` (each with its
    AppendSequence in `seqs`), one event pair around all of them: total ms. The
    lengths are restored outside the graph before each replay."""
    import torch
    dev = xs[0].q.device
    if getattr(dec, "q", None) is None:
        dec.q = torch.empty_like(xs[0].q)
    n = len(xs)

    def step(i):
        xi, a = xs[i % n], seqs[i % n]
        native.rope_append_route(a.q_in[i // n], a.k_new, a.v_new, a.cos, a.sin, a.seq_lens, xi.k_cache,
                                 xi.v_cache, xi.k0, xi.v0, tau, dec.q, dec.route_mask, dec.active_list)
        native.decode_attention(dec.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, a.seq_lens, dec.active_list, dec.out,
                                0, dec.workspace)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):  # eager warm-up outside the capture
        for i in range(min(steps, n)):
            step(i)
    torch.cuda.current_stream(dev).wait_stream(side)
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        e0.record(st)
        for i in range(steps):
            step(i)
        e1.record(st)
    g.sr_events = (e0, e1)  # recorded on every replay: they must live as long as the graph
    for _ in range(max(1, -(-warmup // steps))):  # untimed: warm-up and the graph's launch set-up
        for a in seqs:
            a.reset()
        g.replay()
    torch.cuda.synchronize()
    for a in seqs:
        a.reset()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def _captured_append_steps(native, dec, x, a, tau, steps, flush, split_events):
    """As _captured_steps for the append path: per step an L2 flush and the
    seq_lens reset, then an event, sr_rope_append_route, (an event,)
    sr_decode_attention, an event."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(steps)]
    side = torch.cuda.Stream(device=x.q.device)
    side.wait_stream(torch.cuda.current_stream(x.q.device))
    with torch.cuda.stream(side):
        a.step(native, dec, x, tau)
        flush.sum()
    torch.cuda.current_stream(x.q.device).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        for i in range(steps):
            flush.sum()
            a.seq_lens.copy_(a.seq_saved)
            ev[i][0].record(st)
            native.rope_append_route(a.q_in, a.k_new, a.v_new, a.cos, a.sin, a.seq_lens, x.k_cache, x.v_cache,
                                     x.k0, x.v0, tau, dec.q, dec.route_mask, dec.active_list)
            if split_events:
                ev[i][1].record(st)
            native.decode_attention(dec.q, x.k_cache, x.v_cache, x.k0, x.v0, a.seq_lens, dec.active_list, dec.out,
                                    0, dec.workspace)
            ev[i][2].record(st)
    g.sr_events = ev  # recorded on every replay: they must live as long as the graph
    return g, ev


def time_append(native, dec, x, a, steps, warmup):
    """(step times, prestep kernel times) in ms of the append path."""
    import torch
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=x.q.device)
    gw, _ = _captured_append_steps(native, dec, x, a, x.tau, warmup, flush, False)
    g, ev = _captured_append_steps(native, dec, x, a, x.tau, steps, flush, False)
    gk, evk = _captured_append_steps(native, dec, x, a, x.tau, steps, flush, True)
    gw.replay()
    g.replay()  # untimed: a graph's first replay pays its one-time launch set-up
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    steps_ms = [e[0].elapsed_time(e[2]) for e in ev]
    gk.replay()
    gk.replay()
    torch.cuda.synchronize()
    pre_ms = [e[0].elapsed_time(e[1]) for e in evk]
    del flush
    return steps_ms, pre_ms


def measure_config(native, inputs, name, steps, warmup, flush, device, peak, l2_mode="rotate", copies=None,
                   label=None, **kw):
    """Routed and routing-disabled two-call steps and the fused launch of one more
    workload, K steps back to back per graph. l2_mode: "hot" (the same inputs
    every step, L2-resident when small) or "rotate" (the steps cycle over
    independently seeded input sets whose caches together exceed three times
    L2; `copies` overrides their number)."""
    import torch
    if l2_mode == "hot":
        xs = [inputs.make(name, seed=100, device=device, **kw)]
    elif copies:
        xs = [inputs.make(name, seed=100 + 7919 * c, device=device, **kw) for c in range(copies)]
    else:
        xs = input_sets(inputs, name, 100, device, **kw)
    x = xs[0]
    nobar = lambda: None  # noqa: E731
    r = measure_workload(native, inputs, xs, steps, warmup, flush, nobar, fused=True, isolated=False)
    us, us_dis = r["block"] / steps * 1e3, r["block_disabled"] / steps * 1e3
    us_f, us_fd = r["block_fused"] / steps * 1e3, r["block_fused_disabled"] / steps * 1e3
    need, need_all = r["need"], r["need_all"]
    gbs = need / (us * 1e-6) / 1e9
    acts = [len(a) for a in r["actives"]]
    out = {"workload": label or name, "context": x.max_seq_len,
           "l2": "hot (one input set)" if l2_mode == "hot" else
           f"rotate over {len(xs)} input sets ({len(xs) * x.k_cache.numel() * 4 / 2**30:.2f} GiB of K/V)",
           "us_per_layer_step": round(us, 3), "needed_bytes": int(need), "effective_gbs": round(gbs, 1),
           "frac_of_hbm_peak": round(gbs / peak, 4),
           "active_units": acts[0] if len(set(acts)) == 1 else acts, "units": x.batch * x.n_kv_heads,
           "routing_disabled_us": round(us_dis, 3),
           "routing_disabled_gbs": round(need_all / (us_dis * 1e-6) / 1e9, 1),
           "speedup_routed": round(us_dis / us, 3),
           "fused_us": round(us_f, 3), "fused_disabled_us": round(us_fd, 3),
           "fused_speedup_routed": round(us_fd / us_f, 3)}
    del xs, x, r
    torch.cuda.empty_cache()
    return out


def measure_workload(native, inputs, xs, steps, warmup, flush, barrier, fused=True, isolated=True):
    """Timings of one workload on this GPU. `xs` are input sets of the workload
    (xs[0] the main one) that together exceed L2.

    block*: K layer-steps back to back in one graph over the input sets, one
    event pair around all of them (ms in total): two-call routed and disabled,
    and, if asked, the fused launch routed and disabled.
    two*/route/decode (isolated=True): every step on its own between two events
    after an L2 flush, on xs[0] (ms per step), and the two kernels' own times."""
    import torch
    x = xs[0]
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=x.q.device)
    for _ in range(warmup):
        for xi in xs:
            dec.step(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, xi.tau)
            dec.step_fused(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, xi.tau)
    torch.cuda.synchronize()
    err = dec.workspace.device_error()
    if err:
        raise RuntimeError(f"device error word {err} after warm-up")
    needs, needs_all, acts = [], [], []
    for xi in xs:
        dec.step(xi.q, xi.k_cache, xi.v_cache, xi.k0, xi.v0, xi.seq_lens, xi.tau)
        act = active_units_of(dec.active_list.cpu())
        sl = xi.seq_lens.cpu().tolist()
        needs.append(inputs.needed_bytes(sl, act, xi.n_kv_heads, xi.n_q_heads, xi.batch))
        needs_all.append(inputs.needed_bytes(sl, range(xi.batch * xi.n_kv_heads), xi.n_kv_heads, xi.n_q_heads,
                                             xi.batch))
        acts.append(act)
    # the byte counts of the block are the mean over the rotated sets; the
    # isolated steps run on xs[0]
    r = dict(dec=dec, active=acts[0], actives=acts, need=statistics.mean(needs),
             need_all=statistics.mean(needs_all), need0=needs[0], need_all0=needs_all[0])
    x_tau = x.tau
    r["block"] = time_back_to_back(native, dec, xs, x_tau, steps, warmup, False, barrier)[0]
    r["block_disabled"] = time_back_to_back(native, dec, xs, float("inf"), steps, warmup, False, barrier)[0]
    if fused:
        r["block_fused"] = time_back_to_back(native, dec, xs, x_tau, steps, warmup, True, barrier)[0]
        r["block_fused_disabled"] = time_back_to_back(native, dec, xs, float("inf"), steps, warmup, True,
                                                      barrier)[0]
    if isolated:
        r["two"] = time_steps(native, dec, x, x_tau, steps, warmup, flush, barrier, False)
        r["route"], r["decode"] = time_kernels(native, dec, x, x_tau, steps, flush)
        # the decode kernel under the block's own L2 conditions: events around
        # each decode launch, the steps rotating over the input sets, no flush
        _, r["decode_rot"] = time_kernels(native, dec, x, x_tau, steps, None, rotate=xs)
        r["need_rot"] = [needs[i % len(xs)] for i in range(steps)]
        r["two_disabled"] = time_steps(native, dec, x, float("inf"), steps, warmup, flush, barrier, False)
        if fused:
            r["fused"] = time_steps(native, dec, x, x_tau, steps, warmup, flush, barrier, True)
    err = dec.workspace.device_error()
    if err:
        raise RuntimeError(f"device error word {err} after the timed steps")
    return r


def n_input_sets(x, min_bytes=3 * (126 << 20), max_sets=32) -> int:
    """Input sets to rotate over for workload x: at least three, and as many as
    it takes for their K/V caches together to exceed `min_bytes` (three times
    L2), so that no step finds its inputs in L2."""
    per_set = x.k_cache.numel() * 2 * 2
    return max(3, min(max_sets, -(-min_bytes // per_set)))


def input_sets(inputs, name, seed, device, **kw):
    """n_input_sets independently seeded input sets of one workload."""
    xs = [inputs.make(name, seed=seed, device=device, **kw)]
    xs += [inputs.make(name, seed=seed + 7919 * c, device=device, **kw) for c in range(1, n_input_sets(xs[0]))]
    return xs


def e2e_measure(native, x, steps):
    """Same step through the public API with host buffers: pinned host -> device
    copies of every input, the two calls, and device -> host of the outputs,
    all inside the timed region."""
    import torch
    names = ["q", "k_cache", "v_cache", "k0", "v0", "seq_lens"]
    host = {n: getattr(x, n).cpu().pin_memory() for n in names}
    dev = {n: torch.empty_like(getattr(x, n)) for n in names}
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=x.q.device)
    out_h = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    mask_h = torch.empty(dec.route_mask.shape, dtype=dec.route_mask.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + mask_h.numel()
    st = torch.cuda.current_stream()

    def one():
        for n in names:
            dev[n].copy_(host[n], non_blocking=True)
        dec.step_fused(dev["q"], dev["k_cache"], dev["v_cache"], dev["k0"], dev["v0"], dev["seq_lens"], x.tau)
        out_h.copy_(dec.out, non_blocking=True)
        mask_h.copy_(dec.route_mask, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        one()
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del dev, host
    return ms, h2d, d2h


def _packed_token_inputs(a):
    """The new token's q/k/v projections packed in one pinned host buffer and
    one device buffer (views of each), so that a step moves them with a single
    host -> device copy. Returns (host, device, views on the device)."""
    import torch
    parts = [a.q_in, a.k_new, a.v_new]
    sizes = [t.numel() for t in parts]
    host = torch.empty(sum(sizes), dtype=torch.bfloat16).pin_memory()
    dev = torch.empty(sum(sizes), dtype=torch.bfloat16, device=a.q_in.device)
    views, off = [], 0
    for t, n in zip(parts, sizes):
        host[off:off + n].copy_(t.reshape(-1).cpu())
        views.append(dev[off:off + n].view(t.shape))
        off += n
    return host, dev, views


def e2e_append_measure(native, x, a, steps):
    """The serving view of the same step through the public API: per step only
    the new token's projections (q_in, k_new, v_new) come from pinned host
    memory, the append step and the scan run against the resident cache, and
    the output and route mask go back to the host, all inside the timed region.
    seq_lens is restored on the device each step so that the context stays at
    the workload's length."""
    import torch
    host, dev, (q_in, k_new, v_new) = _packed_token_inputs(a)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=x.q.device)
    out_h = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    mask_h = torch.empty(dec.route_mask.shape, dtype=dec.route_mask.dtype).pin_memory()
    h2d = host.numel() * host.element_size()
    d2h = out_h.numel() * out_h.element_size() + mask_h.numel()
    st = torch.cuda.current_stream()

    def one():
        dev.copy_(host, non_blocking=True)
        a.seq_lens.copy_(a.seq_saved)
        dec.append_step(q_in, k_new, v_new, a.cos, a.sin, x.k_cache, x.v_cache, x.k0, x.v0, a.seq_lens, x.tau)
        out_h.copy_(dec.out, non_blocking=True)
        mask_h.copy_(dec.route_mask, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        one()
    e1.record(st)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def e2e_append_graph_measure(native, x, a, steps):
    """e2e_append with the whole step captured in one CUDA graph (the way a
    decode server replays a layer): per replay the new token's q/k/v copies
    from pinned host memory, the seq_lens reset, the append step and the scan,
    and the copies of the output and mask back to pinned host memory."""
    import torch
    host, dev, (q_in, k_new, v_new) = _packed_token_inputs(a)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=x.q.device)
    out_h = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    mask_h = torch.empty(dec.route_mask.shape, dtype=dec.route_mask.dtype).pin_memory()

    def one():
        dev.copy_(host, non_blocking=True)
        a.seq_lens.copy_(a.seq_saved)
        dec.append_step(q_in, k_new, v_new, a.cos, a.sin, x.k_cache, x.v_cache, x.k0, x.v0, a.seq_lens, x.tau)
        out_h.copy_(dec.out, non_blocking=True)
        mask_h.copy_(dec.route_mask, non_blocking=True)

    side = torch.cuda.Stream(device=x.q.device)
    side.wait_stream(torch.cuda.current_stream(x.q.device))
    with torch.cuda.stream(side):
        one()
    torch.cuda.current_stream(x.q.device).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        one()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / steps


def oracle_threads(n_active: int, group: int) -> int:
    """Threads for the oracle: one per active (unit, query head) pair, capped
    at the host cores."""
    return max(1, min(os.cpu_count() or 1, max(1, n_active * group)))


def oracle_layer_step_us(x_cpu, budget_s, min_reps=1, threads=None):
    """The fp64 oracle, as it stands, on whole layer-steps of this workload,
    with `threads` threads (default: one per active (unit, query head) pair,
    capped at the host cores; the oracle deals whole heads to its threads)."""
    import torch

    import oracle
    tau = float(torch.tensor(x_cpu.tau, dtype=torch.float32))
    mask, active, _ = oracle.route(x_cpu.q, x_cpu.k0, tau)
    n_act = int(active[0])
    if threads is None:
        threads = oracle_threads(n_act, x_cpu.n_q_heads // x_cpu.n_kv_heads)
    reps = 0
    t0 = time.perf_counter()
    while True:
        oracle.routed_attention(x_cpu.q, x_cpu.k_cache, x_cpu.v_cache, x_cpu.k0, x_cpu.v0, x_cpu.seq_lens, tau,
                                n_threads=threads)
        reps += 1
        if reps >= min_reps and time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return el / reps * 1e6, threads, reps, el


def run_ours(args):
    import datetime

    import torch
    import torch.distributed as dist

    from kv_cache_routing_sr_b200 import inputs, native

    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus > 1 needs torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dev, world)

    peak, peak_kind = hbm_peak()
    # fp32 so that torch sums it in place (a pure 256 MiB read; integer sums would
    # first widen the buffer with a 2 GB write).
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    # three (or more) independently seeded input sets whose caches together
    # exceed L2: the timed steps rotate over them, so no step finds its K/V in L2
    xs = input_sets(inputs, args.config, args.seed + 1000 * rank, dev)
    x = xs[0]
    clocks = ClockSampler(local)
    clocks.start()
    t_wall = time.perf_counter()
    r = measure_workload(native, inputs, xs, args.steps, args.warmup, flush, barrier)
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop()

    K = args.steps
    us_step, value = aggregate_us(max_over_ranks(r["block"]), K, world)
    us_dis, _ = aggregate_us(max_over_ranks(r["block_disabled"]), K, world)
    us_fused, _ = aggregate_us(max_over_ranks(r["block_fused"]), K, world)
    us_fused_dis, _ = aggregate_us(max_over_ranks(r["block_fused_disabled"]), K, world)
    us_iso, _ = aggregate_us(max_over_ranks(sum(r["two"])), K, world)
    us_iso_dis, _ = aggregate_us(max_over_ranks(sum(r["two_disabled"])), K, world)
    us_iso_fused, _ = aggregate_us(max_over_ranks(sum(r["fused"])), K, world)
    step_p = [v * 1e3 for v in r["two"]]
    dec_us = statistics.mean(r["decode"]) * 1e3
    route_us = statistics.median(r["route"]) * 1e3
    need, need0 = r["need"], r["need0"]
    gbs = lambda nbytes, us: nbytes / (us * 1e-6) / 1e9  # noqa: E731
    # the decode kernel alone, launch by launch, in back-to-back steps over the
    # rotated input sets: its bytes over its event-timed durations
    dec_rot_us = statistics.mean(r["decode_rot"]) * 1e3
    achieved = sum(r["need_rot"]) / (sum(r["decode_rot"]) * 1e-3) / 1e9
    traffic = profiled_traffic()

    cfg = describe_config(x, len(r["active"]), world)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(us_step / 1e3, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32", "data": "synthetic",
        "config": cfg,
        "path": "sr_route then sr_decode_attention (decode launch overlaps routing: programmatic dependency)",
        "effective_gbs": round(gbs(need, us_step), 1), "frac_of_hbm_peak": round(gbs(need, us_step) / peak, 4),
        "frac_of_nominal_hbm": round(gbs(need, us_step) / NOMINAL_HBM_GBS, 4),
        "needed_bytes_per_step": need,
        "routing_disabled": {"us_per_layer_step": round(us_dis, 3),
                             "effective_gbs": round(gbs(r["need_all"], us_dis), 1),
                             "frac_of_hbm_peak": round(gbs(r["need_all"], us_dis) / peak, 4),
                             "speedup_routed": round(us_dis / us_step, 3),
                             "active_fraction": round(len(r["active"]) / (x.batch * x.n_kv_heads), 4)},
        "fused_single_launch": {"path": "sr_route_decode_attention (every CTA routes in its prologue)",
                                "us_per_layer_step": round(us_fused, 3),
                                "effective_gbs": round(gbs(need, us_fused), 1),
                                "routing_disabled_us": round(us_fused_dis, 3)},
        "isolated_step": {
            "note": "every step alone: L2 flush (a 256 MiB read), event, the step, event; on the first input set. "
                    "Two empty kernels measure about 6 us in this protocol (event and launch latency)",
            "us_per_layer_step": round(us_iso, 3),
            "step_us_p10_p50_p90": [round(statistics.quantiles(step_p, n=10)[i], 3) for i in (0, 4, 8)],
            "effective_gbs": round(gbs(need0, us_iso), 1), "frac_of_hbm_peak": round(gbs(need0, us_iso) / peak, 4),
            "routing_disabled_us": round(us_iso_dis, 3), "speedup_routed": round(us_iso_dis / us_iso, 3),
            "fused_us": round(us_iso_fused, 3),
            "route_kernel_us_median": round(route_us, 3), "decode_kernel_us_mean": round(dec_us, 3)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "decode_kernel<2,2> (persistent split-K scan + sink copy + merge)",
                     "algorithmic_bytes_per_launch": round(statistics.mean(r["need_rot"])),
                     "kernel_us_mean": round(dec_rot_us, 3), "peak_source": f"{peak_kind} HBM copy",
                     "timing": "decode kernel alone: K back-to-back steps in one graph (route, event, decode, "
                               "event) over the rotated input sets, no flush; each event pair around a launch "
                               "adds ~2.6 us of event latency to the kernel's time"},
        "gpu_launches": 2 * K,
        "timing": "value: the K timed layer-steps back to back in one CUDA graph (sr_route, sr_decode_attention, "
                  "per step), one event pair around all of them; the graph is replayed once untimed (the warm-up, "
                  "which also absorbs a graph's one-time launch set-up) and then once timed; the routing-disabled "
                  "and fused figures use the same protocol",
        "clocks": clk,
        "timed_wall_s": round(t_wall, 3),
        "impl": "ours",
    }
    del r
    # The step from un-rotated projections: RoPE + append + capture + route in
    # one launch, then the scan.
    app = AppendInputs(native, inputs, x)
    dec_a = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=dev)
    app_ms, pre_ms = time_append(native, dec_a, x, app, K, args.warmup)
    if dec_a.workspace.device_error():
        raise RuntimeError("device error word set by the append-step timing")
    us_app, _ = aggregate_us(max_over_ranks(sum(app_ms)), K, world)
    # the same step back to back over the rotated input sets, as the headline
    seqs = [AppendSequence(native, inputs, xi, -(-K // len(xs))) for xi in xs]
    ms_b2b = time_append_back_to_back(native, dec_a, xs, seqs, x.tau, K, args.warmup)
    if dec_a.workspace.device_error():
        raise RuntimeError("device error word set by the back-to-back append-step timing")
    us_app_b2b, _ = aggregate_us(max_over_ranks(ms_b2b), K, world)
    line["append_step"] = {
        "path": "sr_rope_append_route then sr_decode_attention (RoPE of the query heads and the new key, KV "
                "append, k0/v0 capture, routing and the length update in the first launch)",
        "us_per_layer_step": round(us_app_b2b, 3),
        "timing": "the K steps back to back in one CUDA graph over the rotated input sets (as value); each set's "
                  "visits append at its last K/sets slots, the last visit at the final slot",
        "isolated_us_per_layer_step": round(us_app, 3),
        "isolated_two_call_us_per_layer_step": round(us_iso, 3),
        "isolated_timing": "L2 flush, event, the two launches, event (as isolated_step), new token at the last slot",
        "prestep_kernel_us_median": round(statistics.median(pre_ms) * 1e3, 3),
        "active_units": int(dec_a.active_list[0])}
    del dec_a, seqs
    if world == 1 and not args.no_sweep:
        sweep = []
        ks = max(20, min(K, 50))
        for frac in (0.0, 0.25, 0.5, 0.75, 1.0):
            x5 = input_sets(inputs, "llama8b_512k", args.seed, dev, sink_fraction=frac)
            s5 = measure_workload(native, inputs, x5, ks, args.warmup, flush, barrier, fused=False)
            u5 = s5["block"] / ks * 1e3
            ud5 = s5["block_disabled"] / ks * 1e3
            d5 = statistics.mean(s5["decode"]) * 1e3
            sweep.append({"sink_fraction": frac, "us_per_layer_step": round(u5, 2),
                          "effective_gbs": round(s5["need"] / (u5 * 1e-6) / 1e9, 1),
                          "frac_of_peak": round(s5["need"] / (u5 * 1e-6) / 1e9 / peak, 4),
                          "decode_kernel_gbs": round(s5["need0"] / (d5 * 1e-6) / 1e9, 1),
                          "routing_disabled_us": round(ud5, 2), "speedup_routed": round(ud5 / u5, 3),
                          "isolated_us": round(statistics.mean(s5["two"]) * 1e3, 2),
                          "isolated_disabled_us": round(statistics.mean(s5["two_disabled"]) * 1e3, 2)})
            del x5, s5
            torch.cuda.empty_cache()
        line["sweep_512k"] = sweep
    if world == 1 and not args.no_sweep:
        # The remaining workloads (K steps back to back per graph): tiny 4K with
        # L2 hot and with its inputs rotated beyond L2, the ragged 70B-shaped and
        # the LLaVA-shaped layers.
        oc_steps = max(20, min(K, 50))
        line["other_configs"] = [
            measure_config(native, inputs, "tiny_4k", oc_steps, args.warmup, flush, dev, peak, "hot"),
            measure_config(native, inputs, "tiny_4k", oc_steps, args.warmup, flush, dev, peak, "rotate"),
            measure_config(native, inputs, "llama70b_ragged", oc_steps, args.warmup, flush, dev, peak),
            measure_config(native, inputs, "llava7b_mha", oc_steps, args.warmup, flush, dev, peak),
        ]
        # Short contexts: the 8B-shaped layer (4 of 8 groups sinks) from 4K to
        # 64K, two-call and fused, routed and disabled, inputs rotated beyond L2.
        short = [measure_config(native, inputs, "llama8b_128k", oc_steps, args.warmup, flush, dev, peak,
                                label=f"llama8b_{c // 1024}k", max_ctx=c)
                 for c in (4096, 8192, 16384, 32768, 65536)]
        faster = ["fused" if e["fused_us"] < e["us_per_layer_step"] else "two-call" for e in short]
        line["short_context"] = {
            "points": short,
            "faster_path": dict(zip([e["workload"] for e in short], faster)),
            "speedup_routed_two_call": {e["workload"]: e["speedup_routed"] for e in short}}
    if not args.no_e2e:
        ms, h2d, d2h = e2e_measure(native, x, args.e2e_steps)
        ms = max_over_ranks(ms)
        line["e2e"] = {"value": round(ms * 1e3 / world, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                       "path": "sr_route_decode_attention, eager launch",
                       "note": "pinned host buffers; every input (caches included) copied each step"}
        ms_a, h2d_a, d2h_a = e2e_append_measure(native, x, app, max(args.e2e_steps, 50))
        ms_a = max_over_ranks(ms_a)
        line["e2e_append"] = {"value": round(ms_a * 1e3 / world, 3), "unit": UNIT, "h2d_bytes_per_step": h2d_a,
                              "d2h_bytes_per_step": d2h_a,
                              "path": "Decoder.append_step, eager launch, KV cache resident",
                              "note": "per step: the new token's q/k/v projections host -> device in one "
                                      "packed copy, the output and route mask device -> host"}
        try:
            ms_g = e2e_append_graph_measure(native, x, app, max(args.e2e_steps, 50))
            failed = 0.0
        except Exception as e:  # capture of the host copies refused: report, do not fail the run
            ms_g, failed, why = 0.0, 1.0, f"{type(e).__name__}: {str(e)[:160]}"
        ms_g, failed = max_over_ranks(ms_g), max_over_ranks(failed)  # same collectives on every rank
        line["e2e_append"]["graph_replay"] = (
            {"value": round(ms_g * 1e3 / world, 3), "unit": UNIT,
             "note": "the same copies and calls captured in one CUDA graph, one replay per step"}
            if not failed else {"unavailable": why if "why" in locals() else "failed on another rank"})
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        xc = x.to("cpu")
        us, threads, reps, el = oracle_layer_step_us(xc, args.cpu_budget_s)
        us1, _, reps1, el1 = oracle_layer_step_us(xc, args.cpu_budget_s / 2, threads=1)
        line["cpu_baseline"] = {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{reps} whole layer-steps of {x.workload.name} "
                                          f"({x.batch * x.n_kv_heads} units) in {el:.1f} s, fp64 C oracle, "
                                          f"{threads} threads (one per active (unit, query head) pair, capped "
                                          f"at the host cores)",
                                "host_cores": os.cpu_count(),
                                "one_thread": {"value": round(us1, 1), "unit": UNIT,
                                               "sample": f"{reps1} layer-steps in {el1:.1f} s"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------------
# reference arm: the oracle on the host cores

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import torch

    from kv_cache_routing_sr_b200 import inputs
    x = inputs.make(args.config, seed=args.seed, device="cpu")
    tau = float(torch.tensor(x.tau, dtype=torch.float32))
    import oracle
    mask, active, _ = oracle.route(x.q, x.k0, tau)
    n_act = int(active[0])
    threads = oracle_threads(n_act, x.n_q_heads // x.n_kv_heads)
    # Each step is one whole layer-step unless that would make the run exceed
    # about three minutes; then a step is a bounded sample of the active units,
    # scaled to the whole layer-step.
    t0 = time.perf_counter()
    oracle.routed_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, tau, n_threads=threads)
    one = time.perf_counter() - t0
    total_steps = args.steps + args.warmup
    units = None
    scale = 1.0
    sample = "whole layer-step"
    if one * total_steps > 180.0 and n_act > 1:
        keep = max(1, int(n_act * 180.0 / (one * total_steps)))
        act = [int(u) for u in active[1:1 + n_act]]
        units = act[:keep]
        scale = n_act / keep
        sample = f"{keep} of {n_act} active units per step, scaled by {scale:.2f}"
    times = []
    for i in range(total_steps):
        t0 = time.perf_counter()
        mask, _, _ = oracle.route(x.q, x.k0, tau)
        oracle.decode(x.q, x.k_cache, x.v_cache, x.v0, x.seq_lens, mask, units=units, n_threads=threads)
        el = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(el * scale)
    us = statistics.mean(times) * 1e6
    line = {
        "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": describe_config(x, n_act, world),
        "impl": "reference",
        "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample + f", fp64 C oracle on {threads} host threads (one per active "
                                            f"(unit, query head) pair, capped at the host cores)",
                         "host_cores": os.cpu_count()},
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """A few eager two-call steps of one workload, for profiler captures: no
    timing, no flush, few launches before the captured ones."""
    import torch

    from kv_cache_routing_sr_b200 import inputs, native
    x = inputs.make(args.profile, seed=args.seed, device="cuda", max_ctx=args.max_ctx)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    for _ in range(args.warmup + args.steps):
        dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    torch.cuda.synchronize()
    if dec.workspace.device_error():
        raise RuntimeError(f"device error word {dec.workspace.device_error()}")
    act = active_units_of(dec.active_list.cpu())
    need = inputs.needed_bytes(x.seq_lens.cpu().tolist(), act, x.n_kv_heads, x.n_q_heads, x.batch)
    print(json.dumps({"profile": args.profile, "batch": x.batch, "context": x.max_seq_len,
                      "q_heads": x.n_q_heads, "kv_heads": x.n_kv_heads, "active_units": len(act),
                      "units": x.batch * x.n_kv_heads, "needed_bytes_per_step": need,
                      "steps": args.warmup + args.steps, "launches_per_step": 2}))


def run_multilayer(args):
    """Per-token attention latency of an n-layer Llama-3.1-8B-shaped stack (each
    layer its own 4-of-8-sinks inputs and cache), one CUDA graph per token."""
    import torch

    from kv_cache_routing_sr_b200 import multilayer
    peak, peak_kind = hbm_peak()
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    rows = []
    for ctx in (131072, 262144, 524288):
        stack = multilayer.LayerStack("llama8b_512k", args.layers, seed=args.seed, max_ctx=ctx,
                                      sink_fraction=0.5)
        res = {"context": ctx, "layers": args.layers}
        for key, gate in (("routed_all_layers", multilayer.LayerGate(0, args.layers - 1)),
                          ("routed_layers_8_to_end", multilayer.LayerGate(8, args.layers - 1)),
                          ("routing_disabled", multilayer.LayerGate(1, 0))):
            g = stack.capture(gate)
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize()
            need = stack.needed_bytes()
            st = torch.cuda.current_stream()
            times = []
            for _ in range(max(5, min(args.steps, 20))):
                flush.sum()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                g.replay()
                e1.record(st)
                e1.synchronize()
                times.append(e0.elapsed_time(e1) * 1e3)
            us = statistics.median(times)
            res[key] = {"us_per_token": round(us, 1), "effective_gbs": round(need / (us * 1e-6) / 1e9, 1),
                        "frac_of_hbm_peak": round(need / (us * 1e-6) / 1e9 / peak, 4),
                        "active_fraction": round(stack.active_fraction(), 4)}
            del g
        res["speedup_all_layers"] = round(res["routing_disabled"]["us_per_token"] /
                                          res["routed_all_layers"]["us_per_token"], 3)
        rows.append(res)
        del stack
        torch.cuda.empty_cache()
    print(json.dumps({"measurement": "per-token attention latency, layer stack in one CUDA graph",
                      "workload": "Llama-3.1-8B-shaped layers (32 q / 8 kv heads, head_dim 128, bf16), batch 1, "
                                  "4 of 8 groups planted sinks per layer, tau 0.6",
                      "peak_gbs": peak, "peak_source": f"{peak_kind} HBM copy", "rows": rows}), flush=True)


def run_proxy_quality(args):
    """Sweep the routing threshold on graded synthetic decode steps (2048 units,
    context 16K) and report precision / recall / F1 against the full-attention
    sink event at three cutoffs."""
    from kv_cache_routing_sr_b200 import inputs, proxy_quality
    taus = [round(0.05 * i, 2) for i in range(0, 20)]
    x = inputs.make_graded(seed=args.seed, batch=256, n_kv_heads=8, group=4, ctx=16384, device="cuda")
    out = {"measurement": "routing proxy vs full-attention sink event (graded synthetic steps)",
           "workload": "batch 256 x 8 KV groups x 4 query heads, context 16384, sink strength t ~ U(0,1)",
           "results": []}
    for cutoff in (0.5, 0.8, 0.95):
        res = proxy_quality.evaluate(x, taus, cutoff=cutoff)
        out["results"].append(res)
    print(json.dumps(out), flush=True)


def run_context_parallel(args):
    """Context-parallel layer-step: every rank scans its shard of the 512K
    sequence, the ranks all-gather their (o, lse) rows and every rank combines
    them. Per step: L2 flush, event, route + partial scan, event, all-gather +
    combine, event; eager launches (the collective stays out of CUDA graphs).
    Time is the max over ranks."""
    import datetime

    import torch
    import torch.distributed as dist

    from kv_cache_routing_sr_b200 import context_parallel as cp
    from kv_cache_routing_sr_b200 import inputs

    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peak, peak_kind = hbm_peak()
    x = inputs.make("llama8b_512k", seed=args.seed, device=dev, sink_fraction=0.5)
    bounds = cp.shard_bounds(x.seq_lens.tolist(), world)
    ks, vs = cp.shard_cache(x.k_cache, bounds[rank]), cp.shard_cache(x.v_cache, bounds[rank])
    lens = torch.tensor([e - s for s, e in bounds[rank]], dtype=torch.int32, device=dev)
    q, k0, v0, tau = x.q, x.k0, x.v0, x.tau
    need = None
    d = cp.ContextParallelDecoder(x.batch, x.n_q_heads, x.n_kv_heads, ks.shape[2], world=world, device=dev)
    d.step(q, ks, vs, k0, v0, lens, tau)
    torch.cuda.synchronize()
    act = active_units_of(d.dec.active_list.cpu())
    need = inputs.needed_bytes(x.seq_lens.tolist(), act, x.n_kv_heads, x.n_q_heads, x.batch)
    del x
    torch.cuda.empty_cache()
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        d.step(q, ks, vs, k0, v0, lens, tau)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st = torch.cuda.current_stream()
    for i in range(K):
        flush.sum()
        ev[i][0].record(st)
        d.local(q, ks, vs, k0, v0, lens, tau)
        ev[i][1].record(st)
        d.finish()
        ev[i][2].record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    tot = [e[0].elapsed_time(e[2]) for e in ev]
    loc = [e[0].elapsed_time(e[1]) for e in ev]
    fin = [e[1].elapsed_time(e[2]) for e in ev]
    err = d.dec.workspace.device_error()
    if err:
        raise RuntimeError(f"device error word {err}")
    us = reduce_max(sum(tot), dev, world) / K * 1e3
    us_loc = reduce_max(sum(loc), dev, world) / K * 1e3
    us_fin = reduce_max(sum(fin), dev, world) / K * 1e3
    if rank == 0:
        gbs = need / (us * 1e-6) / 1e9
        line = {"metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": round(us / 1e3, 6), "higher_is_better": False,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32", "data": "synthetic",
                "config": {"workload": "llama8b_512k", "sink_fraction": 0.5, "batch": 1, "context": 524288,
                           "q_heads": 32, "kv_heads": 8, "head_dim": 128, "tau": 0.6, "active_units": len(act),
                           "parallelism": f"cp{world} (positions sharded; one all-gather of (o, lse) per step)",
                           "l2": "256 MiB read before every step"},
                "mode": "context_parallel", "impl": "ours",
                "effective_gbs": round(gbs, 1), "frac_of_hbm_peak_whole_job": round(gbs / (peak * world), 4),
                "local_us": round(us_loc, 3), "exchange_and_combine_us": round(us_fin, 3),
                "row_bytes_per_rank": d.stride * 4, "timing": "eager launches, CUDA events per step, max over ranks",
                "peak_source": f"{peak_kind} HBM copy"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.context_parallel:
        if args.impl == "reference":
            raise SystemExit("--context-parallel has no reference arm")
        run_context_parallel(args)
        return
    if args.proxy_quality:
        run_proxy_quality(args)
        return
    if args.profile:
        return run_profile(args)
    if args.multilayer:
        run_multilayer(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
