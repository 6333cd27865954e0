"""Benchmark of the gated linear attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                    [--mode forward|backward] [--variant plain|rope|gdn|softmax]

One step = one gla_forward call (increment -> gated scan -> output kernels)
over one batch of the workload, inputs resident in HBM; with --mode backward,
one gla_backward call (d = 128) instead; with --variant, one call of
gla_forward_rope, gla_forward_gdn or gla_softmax_anchor.  With N > 1 (torchrun,
one process per GPU) every rank runs its own independent copy of the workload
(heads and sequences are independent: weak scaling, no data-path
collective); the timed region is bracketed by a barrier and a device
synchronisation and the time is the maximum over ranks.  Rank 0 prints one
JSON line.

`--impl reference` times the fp64 CPU oracle on the host cores instead (one
(batch, head) slice of the workload per step), on rank 0 only.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import (WORKLOADS, gdn_workload, make_beta, make_grads, make_inputs,  # noqa: E402
                       make_state, rope_dims, anchor_workload, make_anchor_gate)

METRIC = "gated linear attention tokens/s (bf16, 720p shapes); % of roofline on 1 B200"
METRIC_BWD = "gated linear attention backward tokens/s (bf16, 720p shapes); % of roofline on 1 B200"


ANCHOR_WINDOW = 2  # softmax anchor: frames in the local window; sinks = the first frame


def anchor_pairs(w, window: int, n_sink: int) -> int:
    """(query, key) pairs of the softmax anchor layer over the whole batch."""
    T = w.tokens_per_frame
    per_bh = 0
    for f in range(w.frames):
        w_lo = max(0, f - window + 1) * T
        per_bh += T * (min(n_sink, w_lo) + (f + 1) * T - w_lo)
    return per_bh * w.B * w.H


def metric_for(mode: str, variant: str) -> str:
    """The metric string of the timed path (the same for both arms)."""
    if mode == "backward":
        return METRIC_BWD
    if variant == "softmax":
        return ("softmax anchor tokens/s (sinks + %d-frame window, bf16, 720p shapes); "
                "%% of roofline on 1 B200" % ANCHOR_WINDOW)
    if variant == "rope":
        return METRIC.replace("attention", "attention + 3D RoPE", 1)
    if variant == "gdn":
        return METRIC.replace("gated linear attention", "frame-wise gated delta rule", 1)
    return METRIC


UNIT = "tokens/s"
DEFAULT_WORKLOAD = "720p-5s"
# An earlier measurement on this GPU type: copy bandwidth, and cuBLAS bf16 as a
# burst and as a seconds-long loop under the 1 kW power cap.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}

# DRAM bytes (read + write) per launch from one ncu capture of each kernel on
# the full workload, valid only while the kernel's sources are unchanged: the
# hash of its files must match.
KERNEL_DEPS = {
    "output": ["gla_output.cuh", "gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "increment": ["gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "scan": ["gla_scan.cuh", "gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "bwd_q": ["gla_bwd_q.cuh", "gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "bwd_kv": ["gla_bwd_kv.cuh", "gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    # the variants' kernels, keyed "<variant>:<kernel>"
    "gdn:increment": ["gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "gdn:output": ["gla_output.cuh", "gla_increment.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "rope:increment": ["gla_increment.cuh", "gla_rope.cuh", "gla_common.cuh", "sm100_ptx.cuh"],
    "rope:output": ["gla_output.cuh", "gla_rope.cuh", "gla_increment.cuh", "gla_common.cuh",
                    "sm100_ptx.cuh"],
    "softmax:anchor": ["gla_softmax_anchor.cuh", "gla_increment.cuh", "gla_common.cuh",
                       "sm100_ptx.cuh"],
}
NCU_TRAFFIC = {
    "720p-5s": {  # ncu, one kernel and one full-size launch per capture
        "increment": (1899706880 + 65776896, "77706b5453f8c685"),
        "scan": (76420096 + 9461760, "dc825921952c30f6"),
        "output": (985888512 + 898614528, "ca0d25760e183b6d"),
        "bwd_q": (1973153536 + 989409536, "b350490e812e8a26"),
        "bwd_kv": (1972606464 + 1851236096, "482f220a22e6fbfc"),
        "gdn:increment": (1899975680 + 130081536, "77706b5453f8c685"),
        "gdn:output": (985748224 + 898199552, "ca0d25760e183b6d"),
        "rope:increment": (1899834880 + 66113536, "57a13fddf495cfb7"),
        "rope:output": (986200576 + 900601088, "8050e870a97585fa"),
        "softmax:anchor": (8292931328 + 944969472, "4c96ba0ee6f65e3e"),
    },
}


# ----------------------------------------------------------------- helpers


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for n in KERNEL_DEPS[kernel]:
        with open(os.path.join(ROOT, "gated_linear_attention_frame_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch measured by ncu for this workload and kernel, or
    None when there is no capture or the kernel changed since."""
    entry = NCU_TRAFFIC.get(workload, {}).get(kernel)
    if entry is None or kernel not in KERNEL_DEPS or entry[1] != kernel_source_hash(kernel):
        return None
    return entry[0]


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS)


def algorithmic_work(w, state_in: bool, state_out: bool = True) -> dict:
    """Bytes and flops the layer must move / compute (no workspace traffic).
    Per token-head: q, k, v read and out written in bf16 = 8d bytes;
    flops 2d(d+1) (increment) + 2d(d+1) (output) + d (divide).
    Per (b, h): state_in read / state_out written, d(d+1) fp32 each.
    Per (b, f, h): one fp32 gate and 2d(d+1) scan flops."""
    d = w.d
    th = w.B * w.tokens * w.H
    bh = w.B * w.H
    units = w.B * w.frames * w.H
    k1_bytes = th * 4 * d
    k3_bytes = th * 4 * d
    k2_bytes = units * 4 + bh * d * (d + 1) * 4 * (int(state_in) + int(state_out))
    flops = th * (4 * d * (d + 1) + d) + units * 2 * d * (d + 1)
    return {"increment": k1_bytes, "scan": k2_bytes, "output": k3_bytes,
            "bytes": k1_bytes + k2_bytes + k3_bytes, "flops": flops}


def algorithmic_work_backward(w, state_in: bool, dstate_out: bool, dstate_in: bool) -> dict:
    """Bytes and flops of the backward pass (no workspace traffic).
    Per token-head, each kernel's own operands in bf16: the recompute's
    increment reads k, v (4d bytes); the query kernel reads q, dout and writes
    dq (6d); the key/value kernel reads k, v and writes dk, dv (8d).  The
    layer's minimum reads q, k, v, dout once and writes dq, dk, dv once (14d).
    Flops per token-head: increment 2d(d+1); [num | den], dq~ and L_f 2d(d+1)
    each; dk~ 2d(d+1), dv 2d^2.  Per (b, f, h): gates and dgate (8 bytes) and
    the scans' 2d(d+1) each way; per (b, h): the fp32 states read / written."""
    d = w.d
    th = w.B * w.tokens * w.H
    bh = w.B * w.H
    units = w.B * w.frames * w.H
    sbytes = bh * d * (d + 1) * 4
    work = {
        "increment": th * 4 * d,
        "scan": units * 4 + sbytes * int(state_in),
        "bwd_q": th * 6 * d,
        "scan_bwd": units * 4 + sbytes * (int(state_in) + int(dstate_out) + int(dstate_in)),
        "dgate": units * 8,
        "bwd_kv": th * 8 * d,
    }
    work["bytes"] = th * 14 * d + units * 8 + sbytes * (int(state_in) + int(dstate_out) +
                                                         int(dstate_in))
    work["flops"] = th * (10 * d * (d + 1) + 2 * d * d) + units * 4 * d * (d + 1)
    return work


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read only)
    in a background thread while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML unavailable: report no clocks
            self.ok = False
        self._t = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                pw = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception:
                pass
            self._stop.wait(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self) -> dict | None:
        if not self.ok:
            return None
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sm = [s[0] for s in self.samples]
        mask = 0
        for s in self.samples:
            mask |= int(s[1])
        reasons = [n for n, b in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "power_w_max": round(max(s[2] for s in self.samples), 1)}


# ------------------------------------------------------------ distributed


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(world: int, backend: str):
    if world <= 1:
        return None
    import torch.distributed as dist

    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(x: float, dist, device) -> float:
    """Maximum of a float over ranks (identity without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is None:
        return
    if device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


# --------------------------------------------------------------- CPU oracle


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def oracle_head_slices(w, heads, seed_device="cpu"):
    """Host copies of (q, k, v, g) for the sampled (b, h) slices of call 0."""
    q, k, v, g = make_inputs(w, device=seed_device)
    out = []
    for (b, h) in heads:
        out.append(tuple(x.cpu() for x in (q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h])))
    del q, k, v, g
    return out


def oracle_head_call(w, variant: str):
    """The fp64 oracle of one (b, h) slice for the layer or a variant:
    (workload whose inputs it takes, f(q, k, v, g, b, h, s_in_bh), label)."""
    import oracle

    if variant == "rope":
        def f(q, k, v, g, b, h, s):
            oracle.gla_rope_head(q, k, v, g, w.tokens_per_frame, w.grid_w, 0, rope_dims(w.d),
                                 10000.0, s, w.eps)
        return w, f, "3D-RoPE oracle"
    if variant == "softmax":
        wa = anchor_workload(w)
        z = make_anchor_gate(wa)

        def f(q, k, v, g, b, h, s):
            oracle.softmax_anchor_head(q, k, v, wa.tokens_per_frame, ANCHOR_WINDOW,
                                       wa.tokens_per_frame, z[b, :, h])
        return wa, f, "softmax-anchor oracle"
    if variant == "gdn":
        wg = gdn_workload(w)
        beta = make_beta(wg)

        def f(q, k, v, g, b, h, s):
            oracle.gla_gdn_head(q, k, v, g, beta[b, :, h], wg.tokens_per_frame, s, wg.eps)
        return wg, f, "delta-rule oracle"

    def f(q, k, v, g, b, h, s):
        oracle.gla_head(q, k, v, g, w.tokens_per_frame, s, w.eps)
    return w, f, "oracle"


def time_oracle(w, budget_s: float, max_heads: int | None = None, device="cpu",
                variant: str = "plain") -> dict:
    """Time the fp64 oracle (of the layer or of the variant) on (b, h) slices
    of the workload until `budget_s` of CPU work has been done; tokens/s
    counts full-layer tokens (all heads)."""
    w, head_fn, label = oracle_head_call(w, variant)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    if max_heads:
        pairs = pairs[:max_heads]
    slices = oracle_head_slices(w, pairs[: min(len(pairs), 8)], device)
    s_in = make_state(w)
    done = 0
    t0 = time.perf_counter()
    while True:
        i = done % len(slices)
        b, h = pairs[i]
        q, k, v, g = slices[i]
        head_fn(q, k, v, g, b, h, None if s_in is None else s_in[b, h])
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= 4 * len(pairs):
            break
    tokens = done * w.tokens / w.H * 1.0  # head-slices -> full-layer tokens
    return {"value": tokens / el, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": "%d (batch, head) slices of %s (%d frames x %d tokens each), fp64 numpy "
                      "%s, %.1f s wall" % (done, w.name, w.frames, w.tokens_per_frame, label, el),
            "seconds": round(el, 3)}


# ---------------------------------------------------------------- GPU arm


def e2e_pipelined(dev, stream, dist, world, host_in, dev_out, call, E, tokens):
    """End-to-end metric through the public API with host buffers.  Each of E
    steps copies `host_in` (pinned; None entries pass through as None) to
    device buffers, runs `call(inputs, outputs)` on `stream` and copies the
    outputs back to pinned host buffers, all inside the timed region.  Steps
    are pipelined over three streams (H2D, compute, D2H) with double-buffered
    device buffers, so step i+1's upload overlaps step i's compute and
    download."""
    host_out = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in dev_out]
                for _ in range(2)]
    dbuf = [[None if x is None else torch.empty(x.shape, dtype=x.dtype, device=dev)
             for x in host_in] for _ in range(2)]
    dout = [dev_out, [torch.empty_like(o) for o in dev_out]]
    h2d = sum(x.numel() * x.element_size() for x in host_in if x is not None)
    d2h = sum(o.numel() * o.element_size() for o in dev_out)
    s_h2d = torch.cuda.Stream(dev)
    s_d2h = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b uploaded
    ev_done = [torch.cuda.Event() for _ in range(2)]  # call on buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # results of buffer b downloaded

    def step(i):
        bb = i % 2
        with torch.cuda.stream(s_h2d):
            if i >= 2:
                s_h2d.wait_event(ev_done[bb])  # buffer bb's previous call has read it
            for d_, h_ in zip(dbuf[bb], host_in):
                if h_ is not None:
                    d_.copy_(h_, non_blocking=True)
            ev_in[bb].record(s_h2d)
        stream.wait_event(ev_in[bb])
        if i >= 2:
            stream.wait_event(ev_out[bb])  # buffer bb's previous results downloaded
        call(dbuf[bb], dout[bb])
        ev_done[bb].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_done[bb])
            for h_, d_ in zip(host_out[bb], dout[bb]):
                h_.copy_(d_, non_blocking=True)
            ev_out[bb].record(s_d2h)

    for i in range(2):  # warm the path
        step(i)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    for i in range(E):
        step(i)
    stream.wait_event(ev_out[(E - 1) % 2])
    stream.wait_event(ev_out[E % 2])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = reduce_max(e0.elapsed_time(e1), dist, dev) / E
    return {"value": round(world * tokens / (e_ms * 1e-3), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": E,
            "ms_per_step": round(e_ms, 3),
            "note": "pinned host buffers; H2D, call and D2H pipelined over 3 streams"}


def run_gpu(args, w, dist, rank, local_rank, world):
    import gated_linear_attention_frame_b200 as gla

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()

    rope = args.variant == "rope"
    gdn = args.variant == "gdn"
    if gdn:
        w = gdn_workload(w)  # keys scaled by 1/sqrt(d T): the delta recurrence contracts
        beta_l = make_beta(w, device=dev)
    # inputs: a ring of input sets (fresh frames for the streaming workload)
    nsets = 4 if w.name == "stream" else 1
    sets = [make_inputs(w, call=c, device=dev) for c in range(nsets)]
    state = make_state(w, device=dev)
    state_buf = state.clone() if state is not None else None
    out = torch.empty_like(sets[0][0])
    so = torch.empty(w.B, w.H, w.d, w.d + 1, device=dev, dtype=torch.float32)
    work = algorithmic_work(w, state_in=state is not None)

    def step(i, events=None):
        q, k, v, g = sets[i % nsets]
        s_in = state_buf  # streaming: the state carries from call to call
        s_out = state_buf if state_buf is not None else so
        a = (q, k, v, g, s_in, s_out, out, w.B, w.H, w.frames, w.tokens_per_frame, w.d, w.eps)
        if rope:
            # a carried state advances the temporal position call by call
            off = (i * w.frames) % (1 << 20) if state_buf is not None else 0
            cfg = gla.rope_config(w.grid_w, rope_dims(w.d), off)
            if events is None:
                gla.gla_forward_rope(*a, cfg, stream)
            else:
                gla.gla_forward_rope_timed(*a, cfg, stream, events)
        elif gdn:
            ag = a[:4] + (beta_l,) + a[4:]
            if events is None:
                gla.gla_forward_gdn(*ag, stream)
            else:
                gla.gla_forward_gdn_timed(*ag, stream, events)
        elif events is None:
            gla.gla_forward(*a, stream)
        else:
            gla.gla_forward_timed(*a, stream, events)

    warm = max(3, args.warmup)
    for i in range(warm):
        step(i)
    torch.cuda.synchronize(dev)
    assert gla.gla_device_fault(stream) == 0

    K = args.steps
    # Timed region 1 (the reported value): K plain calls, events around them.
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with clocks:
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    total_ms = reduce_max(t0.elapsed_time(t1), dist, dev)
    ms_step = total_ms / K
    value = world * w.total_tokens / (ms_step * 1e-3)

    # Timed region 2: the same K calls with events recorded between the three
    # kernels on the launching stream (per-kernel durations for the roofline).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for e4 in evs:
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    for i in range(K):
        step(i, evs[i])
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    fault = gla.gla_device_fault(stream)
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
                    for e in evs])

    names = ["increment", "scan", "output"]
    avg = per.mean(axis=0)
    dom = int(np.argmax(avg))
    achieved = work[names[dom]] / (avg[dom] * 1e-3) / 1e9
    traffic = ncu_traffic(w.name, names[dom] if args.variant == "plain"
                          else "%s:%s" % (args.variant, names[dom]))
    roof = {"bound": "hbm", "kernel": "gla_%s_kernel" % names[dom], "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read + write)",
            "algorithmic_bytes_per_launch": work[names[dom]],
            "peak_source": peaks["source"] + " (hbm_gbs)"}
    t_roof = max(work["bytes"] / (peaks["hbm_gbs"] * 1e9),
                 work["flops"] / (peaks["bf16_tflops"] * 1e12))
    layer = {"algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"],
             "roofline_ms": round(t_roof * 1e3, 4), "frac": round(t_roof * 1e3 / ms_step, 4),
             "achieved_GBps": round(work["bytes"] / (ms_step * 1e-3) / 1e9, 1),
             "kernel_ms": {n: round(float(a), 4) for n, a in zip(names, avg)},
             "kernel_ms_note": "per-kernel means from a second pass of K calls with events "
                               "between the kernels"}

    # End to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory, runs the call and copies out and
    # state_out back, all inside the timed region.
    e2e = None
    if not args.no_e2e:
        host_in = [x.cpu().pin_memory() for x in sets[0]]
        host_in.append(state_buf.cpu().pin_memory() if state_buf is not None else None)
        host_in.append(beta_l.cpu().pin_memory() if gdn else None)
        dev_out = [out, so]

        def call(bi, bo):
            q_, k_, v_, g_, s_, b_ = bi
            a = (q_, k_, v_, g_, s_, bo[1], bo[0], w.B, w.H, w.frames, w.tokens_per_frame, w.d,
                 w.eps)
            if rope:
                gla.gla_forward_rope(*a, gla.rope_config(w.grid_w, rope_dims(w.d)), stream)
            elif gdn:
                gla.gla_forward_gdn(*(a[:4] + (b_,) + a[4:]), stream)
            else:
                gla.gla_forward(*a, stream)

        e2e = e2e_pipelined(dev, stream, dist, world, host_in, dev_out, call,
                            max(2, min(K, args.e2e_steps)), w.total_tokens)

    # kernels per call: increment, scan, output; + the rotary table kernel; +
    # the Gram reduction when the tile schedule has tail units (delta rule)
    units = w.B * w.frames * w.H
    ctas = min(units * -(-w.tokens_per_frame // 128),
               torch.cuda.get_device_properties(dev).multi_processor_count)
    launches_per_step = 3 + int(rope) + int(gdn and ctas > 0 and units % ctas != 0)
    metric = metric_for("forward", args.variant)
    res = {
        "metric": metric,
        "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": warm, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "frames": w.frames,
                   "tokens_per_frame": w.tokens_per_frame, "tokens_per_step_per_gpu": w.total_tokens,
                   "state_in": "carried fp32" if state is not None else "zero",
                   "l2": "inputs larger than L2 (%.2f GB read+written per step); no flush"
                         % (work["bytes"] / 1e9),
                   "parallelism": "dp%d (independent sequences per GPU)" % world,
                   **({"rope": {"grid_w": w.grid_w, "dims": list(rope_dims(w.d)),
                                "theta": 10000.0}} if rope else {}),
                   **({"keys": "N(0,1)/sqrt(d T)", "beta_logits": "N(0,1)"} if gdn else {})},
        "roofline": roof, "layer_roofline": layer,
        "gpu_launches": launches_per_step * K,
        "e2e": e2e,
        "clocks": clocks.summary(), "device_fault": fault,
        "gpu": torch.cuda.get_device_name(dev),
    }
    return res


# The other layer workloads timed beside the headline one by the default run
# (same --steps / --warmup; the streaming workload as its 64 consecutive calls
# with the state carried).  The tiny workload is launch-bound: parity only.
OTHER_WORKLOADS = ("480p-5s", "720p-60s", "stream")
STREAM_CALLS = 64


def workload_summary(r: dict) -> dict:
    lr = r["layer_roofline"]
    return {"ms_per_call": r["ms_per_step"], "tokens_per_s": r["value"], "calls": r["steps"],
            "layer_roofline_ms": lr["roofline_ms"], "layer_roofline_frac": lr["frac"],
            "kernel_ms": lr["kernel_ms"], "dominant_kernel": r["roofline"]["kernel"],
            "dominant_kernel_frac": r["roofline"]["frac"],
            "state_in": r["config"]["state_in"], "clocks": r["clocks"],
            "device_fault": r["device_fault"]}


def run_other_workloads(args, head: dict, dist, rank, local_rank, world) -> dict:
    """Every layer workload's line (the headline's included) for one JSON key."""
    out = {head["config"]["workload"]: workload_summary(head)}
    for name in OTHER_WORKLOADS:
        a = argparse.Namespace(**vars(args))
        a.no_e2e = True
        if name == "stream":
            a.steps = STREAM_CALLS
        torch.cuda.empty_cache()
        out[name] = workload_summary(run_gpu(a, WORKLOADS[name], dist, rank, local_rank, world))
    out["tiny"] = "parity only (launch-bound)"
    return out


# The library's other paths at the headline workload, timed by the default run
# as well (fewer steps: each is one call of its entry point per step).
OTHER_PATHS = (("backward", "plain"), ("backward", "saved"), ("forward", "rope"),
               ("forward", "gdn"), ("forward", "softmax"))
PATH_STEPS = 10


def path_summary(r: dict) -> dict:
    out = {"metric": r["metric"], "ms_per_call": r["ms_per_step"], "tokens_per_s": r["value"],
           "calls": r["steps"], "roofline": {k: r["roofline"][k] for k in
                                             ("bound", "kernel", "achieved", "unit", "frac")},
           "layer_roofline_frac": r["layer_roofline"]["frac"], "clocks": r["clocks"],
           "device_fault": r["device_fault"]}
    if "kernel_ms" in r["layer_roofline"]:
        out["kernel_ms"] = r["layer_roofline"]["kernel_ms"]
    if "rollout_step" in r:
        out["rollout_step"] = r["rollout_step"]
    if "saved_context" in r:
        out["saved_context"] = r["saved_context"]
    return out


def run_other_paths(args, w, dist, rank, local_rank, world) -> dict:
    out = {}
    for mode, variant in OTHER_PATHS:
        a = argparse.Namespace(**vars(args))
        a.no_e2e = True
        a.mode, a.variant = mode, "plain" if variant == "saved" else variant
        a.saved = variant == "saved"
        a.steps = min(args.steps, PATH_STEPS)
        torch.cuda.empty_cache()
        if mode == "backward":
            r = run_gpu_backward(a, w, dist, rank, local_rank, world)
        elif variant == "softmax":
            r = run_gpu_anchor(a, w, dist, rank, local_rank, world)
        else:
            r = run_gpu(a, w, dist, rank, local_rank, world)
        key = ("backward_saved" if variant == "saved" else "backward") if mode == "backward" \
            else variant
        out[key] = path_summary(r)
    return out


def run_gpu_backward(args, w, dist, rank, local_rank, world):
    """One step = one gla_backward call over one batch of the workload
    (recompute of the forward states, then the five gradient kernels), or with
    --saved one gla_backward_saved call from the context a gla_forward_train
    call of the same inputs wrote before the timed region (four kernels)."""
    import gated_linear_attention_frame_b200 as gla

    saved_mode = bool(getattr(args, "saved", False))
    if w.d != 128:
        raise SystemExit("the backward pass is built for d = 128")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    q, k, v, g = make_inputs(w, device=dev)
    s_in = make_state(w, device=dev)
    dout, ds_out = make_grads(w, device=dev, dstate_out=s_in is not None)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty_like(g)
    ds_in = torch.empty(w.B, w.H, w.d, w.d + 1, device=dev) if s_in is not None else None
    work = algorithmic_work_backward(w, s_in is not None, ds_out is not None, ds_in is not None)
    saved = None
    fwd_train = None
    if saved_mode:
        saved = torch.empty(max(1, gla.gla_saved_bytes(w.B, w.H, w.frames, w.tokens_per_frame,
                                                       w.d)), device=dev, dtype=torch.uint8)
        f_out = torch.empty_like(q)
        f_state = torch.empty(w.B, w.H, w.d, w.d + 1, device=dev)
        fa = (q, k, v, g, s_in, f_state, f_out)
        dims = (w.B, w.H, w.frames, w.tokens_per_frame, w.d, w.eps, stream)
        # the training forward's cost over the plain forward (context writes)
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for _ in range(3):
            gla.gla_forward(*fa, *dims)
            gla.gla_forward_train(*fa, saved, *dims)
        fe[0].record(stream)
        for _ in range(5):
            gla.gla_forward(*fa, *dims)
        fe[1].record(stream)
        fe[2].record(stream)
        for _ in range(5):
            gla.gla_forward_train(*fa, saved, *dims)
        fe[3].record(stream)
        torch.cuda.synchronize(dev)
        fwd_train = {"forward_ms": round(fe[0].elapsed_time(fe[1]) / 5, 5),
                     "forward_train_ms": round(fe[2].elapsed_time(fe[3]) / 5, 5),
                     "saved_bytes": int(saved.numel()),
                     "note": "the context is written by gla_forward_train before the timed "
                             "region; the timed calls are gla_backward_saved"}

    def step(events=None):
        a = (q, k, v, g, s_in, dout, ds_out, dq, dk, dv, dg, ds_in, w.B, w.H, w.frames,
             w.tokens_per_frame, w.d, w.eps, stream)
        if saved_mode:
            b = a[:5] + (saved,) + a[5:]
            if events is None:
                gla.gla_backward_saved(*b)
            else:
                gla.gla_backward_saved_timed(*b, events)
        elif events is None:
            gla.gla_backward(*a)
        else:
            gla.gla_backward_timed(*a, events)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_device_fault(stream) == 0

    K = args.steps
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with clocks:
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_step = reduce_max(t0.elapsed_time(t1), dist, dev) / K
    value = world * w.total_tokens / (ms_step * 1e-3)

    names = ["increment", "scan", "bwd_q", "scan_bwd", "dgate", "bwd_kv"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(K)]
    for e7 in evs:
        for e in e7:
            e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    fault = gla.gla_device_fault(stream)
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(6)] for e in evs])
    avg = per.mean(axis=0)
    if saved_mode:
        names = names[2:]
        avg = avg[2:]
    dom = int(np.argmax(avg))
    achieved = work[names[dom]] / (avg[dom] * 1e-3) / 1e9
    traffic = ncu_traffic(w.name, names[dom]) if names[dom] in KERNEL_DEPS else None
    roof = {"bound": "hbm", "kernel": "gla_%s_kernel" % names[dom], "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read + write)",
            "algorithmic_bytes_per_launch": work[names[dom]],
            "peak_source": peaks["source"] + " (hbm_gbs)"}
    t_roof = max(work["bytes"] / (peaks["hbm_gbs"] * 1e9),
                 work["flops"] / (peaks["bf16_tflops"] * 1e12))
    layer = {"algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"],
             "roofline_ms": round(t_roof * 1e3, 4), "frac": round(t_roof * 1e3 / ms_step, 4),
             "achieved_GBps": round(work["bytes"] / (ms_step * 1e-3) / 1e9, 1),
             "kernel_ms": {n: round(float(a), 4) for n, a in zip(names, avg)},
             "kernel_ms_note": "per-kernel means from a second pass of K calls with events "
                               "between the kernels"}

    e2e = None
    if not args.no_e2e:
        host_in = [x.cpu().pin_memory() for x in (q, k, v, g, dout)]
        host_in += [None if x is None else x.cpu().pin_memory() for x in (s_in, ds_out)]
        dev_out = [dq, dk, dv, dg] + ([ds_in] if ds_in is not None else [])

        def call(bi, bo):
            q_, k_, v_, g_, do_, s_, dso_ = bi
            tail = (bo[0], bo[1], bo[2], bo[3], bo[4] if len(bo) > 4 else None, w.B, w.H,
                    w.frames, w.tokens_per_frame, w.d, w.eps, stream)
            if saved_mode:  # the context stays on the device, as in training
                gla.gla_backward_saved(q_, k_, v_, g_, s_, saved, do_, dso_, *tail)
            else:
                gla.gla_backward(q_, k_, v_, g_, s_, do_, dso_, *tail)

        e2e = e2e_pipelined(dev, stream, dist, world, host_in, dev_out, call,
                            max(2, min(K, args.e2e_steps)), w.total_tokens)

    res = {
        "metric": METRIC_BWD, "mode": "backward_saved" if saved_mode else "backward",
        "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": warm, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "frames": w.frames,
                   "tokens_per_frame": w.tokens_per_frame, "tokens_per_step_per_gpu": w.total_tokens,
                   "state_in": "fp32 with dstate_out" if s_in is not None else "zero",
                   "l2": "inputs larger than L2 (%.2f GB read+written per step); no flush"
                         % (work["bytes"] / 1e9),
                   "parallelism": "dp%d (independent sequences per GPU)" % world},
        "roofline": roof, "layer_roofline": layer, "gpu_launches": (4 if saved_mode else 6) * K,
        "e2e": e2e, "clocks": clocks.summary(), "device_fault": fault,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if fwd_train is not None:
        res["saved_context"] = fwd_train
    return res


def run_gpu_anchor(args, w, dist, rank, local_rank, world):
    """One step = one gla_softmax_anchor call (sinks = the first frame, a
    window of ANCHOR_WINDOW frames, sigmoid output gate) over one batch."""
    import gated_linear_attention_frame_b200 as gla

    if w.d != 128:
        raise SystemExit("the softmax anchor kernel is built for d = 128")
    w = anchor_workload(w)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    q, k, v, _ = make_inputs(w, device=dev)
    z = make_anchor_gate(w, device=dev)
    out = torch.empty_like(q)
    T, W = w.tokens_per_frame, ANCHOR_WINDOW
    pairs = anchor_pairs(w, W, T)
    flops = 4 * w.d * pairs                         # Q K^T and P V
    nbytes = w.B * w.tokens * w.H * w.d * 2 * 5     # q, k, v, z read; out written

    def step(events=None):
        a = (q, k, v, z, out, w.B, w.H, w.frames, T, w.d, W, T)
        if events is None:
            gla.gla_softmax_anchor(*a, stream)
        else:
            gla.gla_softmax_anchor_timed(*a, stream, events)

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_device_fault(stream) == 0
    K = args.steps
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier(dist, dev)
    torch.cuda.synchronize(dev)
    with clocks:
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_step = reduce_max(t0.elapsed_time(t1), dist, dev) / K
    fault = gla.gla_device_fault(stream)
    achieved = flops / (ms_step * 1e-3) / 1e12
    # the calls run back to back for seconds: the sustained (power-capped)
    # bf16 peak is the denominator, the burst one is reported beside it
    peak = peaks["bf16_tflops_sustained"]
    roof = {"bound": "tensor", "kernel": "gla_softmax_anchor_kernel", "achieved": round(achieved, 1),
            "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": ncu_traffic(w.name, "softmax:anchor"),
            "traffic_unit": "bytes per launch (ncu dram read + write)",
            "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4),
            "algorithmic_flops_per_launch": flops,
            "flops_note": "4 d per (query, key) pair (Q K^T and P V, one online pass)",
            "peak_source": peaks["source"] + " (bf16_tflops_sustained)"}
    t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peak * 1e12))
    layer = {"algorithmic_bytes": nbytes, "algorithmic_flops": flops,
             "roofline_ms": round(t_roof * 1e3, 4), "frac": round(t_roof * 1e3 / ms_step, 4)}
    e2e = None
    if not args.no_e2e:
        host_in = [x.cpu().pin_memory() for x in (q, k, v, z)]

        def call(bi, bo):
            gla.gla_softmax_anchor(bi[0], bi[1], bi[2], bi[3], bo[0], w.B, w.H, w.frames, T,
                                   w.d, W, T, stream)

        e2e = e2e_pipelined(dev, stream, dist, world, host_in, [out], call,
                            max(2, min(K, args.e2e_steps)), w.total_tokens)
    # One rollout step (gla_softmax_anchor_step): the last frame from its sink
    # and window caches, the same K step / warm-up counts, events around them.
    fl = w.frames - 1
    lo = max(0, fl - W + 1)
    rows = slice(fl * T, (fl + 1) * T)
    qs, ks, vs, zs = (x[:, rows].contiguous() for x in (q, k, v, z))
    sk, sv = k[:, :T].contiguous(), v[:, :T].contiguous()
    wk = k[:, lo * T:fl * T].contiguous() if fl > lo else None
    wv = v[:, lo * T:fl * T].contiguous() if fl > lo else None
    os_ = torch.empty_like(qs)

    def rstep():
        gla.gla_softmax_anchor_step(qs, ks, vs, zs, sk, sv, wk, wv, os_, w.B, w.H, T, w.d, fl, W, T,
                                    stream)

    for _ in range(warm):
        rstep()
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    t0.record(stream)
    for _ in range(K):
        rstep()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    ms_r = reduce_max(t0.elapsed_time(t1), dist, dev) / K
    keys_r = min(T, lo * T) + (fl + 1 - lo) * T
    flops_r = 4 * w.d * w.B * w.H * T * keys_r
    rollout = {"call": "gla_softmax_anchor_step", "frame": fl, "keys_per_query": keys_r,
               "ms_per_step": round(ms_r, 5),
               "tokens_per_s": round(world * w.B * T / (ms_r * 1e-3), 1),
               "achieved_tflops": round(flops_r / (ms_r * 1e-3) / 1e12, 1),
               "frac": round(flops_r / (ms_r * 1e-3) / 1e12 / peak, 4),
               "device_fault": gla.gla_device_fault(stream)}
    return {
        "metric": metric_for("forward", "softmax"), "value": round(world * w.total_tokens /
                                                                 (ms_step * 1e-3), 1),
        "unit": UNIT, "n_gpus": world, "steps": K, "warmup": warm,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "frames": w.frames,
                   "tokens_per_frame": T, "window_frames": W, "n_sink": T, "gate": True,
                   "tokens_per_step_per_gpu": w.total_tokens,
                   "l2": "inputs larger than L2; no flush",
                   "parallelism": "dp%d (independent sequences per GPU)" % world},
        "roofline": roof, "layer_roofline": layer, "gpu_launches": K, "e2e": e2e,
        "clocks": clocks.summary(), "device_fault": fault, "rollout_step": rollout,
        "gpu": torch.cuda.get_device_name(dev),
    }


def time_oracle_backward(w, budget_s: float) -> dict:
    """Time the fp64 gradient oracle on (b, h) slices until `budget_s` of CPU
    work; tokens/s counts full-layer tokens (all heads)."""
    import oracle

    pairs = [(b, h) for b in range(w.B) for h in range(w.H)][:4]
    slices = oracle_head_slices(w, pairs)
    dout, _ = make_grads(w)
    douts = [dout[b, :, h].clone() for (b, h) in pairs]
    del dout
    done = 0
    t0 = time.perf_counter()
    while True:
        i = done % len(pairs)
        q, k, v, g = slices[i]
        oracle.gla_backward_head_manual(q, k, v, g, w.tokens_per_frame, douts[i], None, None,
                                        w.eps)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": done * w.tokens / w.H / el, "unit": UNIT, "cores": cpu_threads(),
            "kind": "oracle",
            "sample": "%d (batch, head) slices of %s (%d frames x %d tokens each), fp64 numpy "
                      "gradient oracle, %.1f s wall" % (done, w.name, w.frames,
                                                        w.tokens_per_frame, el),
            "seconds": round(el, 3)}


def run_reference(args, w):
    """fp64 CPU oracle of the timed path (the layer, a variant or the
    gradients), one (batch, head) slice per step."""
    import oracle

    backward = args.mode == "backward"
    w, head_fn, label = oracle_head_call(w, "plain" if backward else args.variant)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    slices = oracle_head_slices(w, pairs[:4])
    s_in = make_state(w)
    if backward:
        dout, _ = make_grads(w)
        douts = [dout[b, :, h].clone() for (b, h) in pairs[:4]]
        del dout

    def step(i):
        b, h = pairs[i % 4]
        q, k, v, g = slices[i % 4]
        if backward:
            oracle.gla_backward_head_manual(q, k, v, g, w.tokens_per_frame, douts[i % 4], None,
                                            None, w.eps)
        else:
            head_fn(q, k, v, g, b, h, None if s_in is None else s_in[b, h])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = args.steps * w.tokens / w.H / el
    sample = ("one (batch, head) slice of %s per step (%d frames x %d tokens), fp64 numpy %s"
              % (w.name, w.frames, w.tokens_per_frame,
                 "gradient oracle" if backward else label))
    return {
        "impl": "reference", "metric": metric_for(args.mode, args.variant), "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "frames": w.frames,
                   "tokens_per_frame": w.tokens_per_frame},
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": cpu_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--mode", choices=["forward", "backward"], default="forward",
                    help="time gla_forward (the layer metric) or gla_backward")
    ap.add_argument("--saved", action="store_true",
                    help="--mode backward: time gla_backward_saved from a gla_forward_train "
                         "context instead of gla_backward (no recompute)")
    ap.add_argument("--variant", choices=["plain", "rope", "gdn", "softmax"], default="plain",
                    help="forward only: the plain layer, gla_forward_rope (3D RoPE), "
                         "gla_forward_gdn (frame-wise gated delta rule) or gla_softmax_anchor")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--frames", type=int, default=0,
                    help="override the workload's frame count (small profiling cases)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (the default run also times the other layer "
                         "workloads into the line's 'workloads' key and the backward pass, "
                         "RoPE, delta-rule and softmax-anchor paths into 'paths')")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for cpu_baseline (0 = skip)")
    args = ap.parse_args(argv)
    w = WORKLOADS[args.workload]
    if args.frames > 0:
        w = w.with_(frames=args.frames, name="%s-%dframes" % (w.name, args.frames))
    rank, local_rank, world = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    if world != args.gpus and world > 1:
        print("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world), file=sys.stderr)
    dist = dist_init(world, "nccl")
    try:
        if args.mode == "backward":
            res = run_gpu_backward(args, w, dist, rank, local_rank, world)
        elif args.variant == "softmax":
            res = run_gpu_anchor(args, w, dist, rank, local_rank, world)
        else:
            res = run_gpu(args, w, dist, rank, local_rank, world)
            if (args.variant == "plain" and args.workload == DEFAULT_WORKLOAD and args.frames == 0
                    and not args.no_workloads):
                res["workloads"] = run_other_workloads(args, res, dist, rank, local_rank, world)
                res["paths"] = run_other_paths(args, w, dist, rank, local_rank, world)
        if rank == 0 and world == 1 and args.cpu_budget > 0:
            res["cpu_baseline"] = (time_oracle_backward(w, args.cpu_budget)
                                   if args.mode == "backward"
                                   else time_oracle(w, args.cpu_budget, variant=args.variant))
        elif rank == 0:
            res["cpu_baseline"] = None
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
