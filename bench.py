#!/usr/bin/env python
"""Benchmark of the FlowCache per-step hot path on B200.

One step = the whole hot path over one layer's synthetic inputs, all through
the libflowcache C-ABI:
  gate (fused Euler update + per-chunk relative L1 + accumulator) over every
  chunk, then importance, redundancy, pooled score + top-B, and K/V compaction
  over every head.
Default workload: the long-history layer (H=40, d=128, L_q=8192, L_k=131072,
B=32768, lambda=0.5, pool 7, bf16, 25% exact duplicate keys; no gate), the
largest configuration that fits one GPU.  The same JSON line carries the full
step of the full-step sweep at L_k=128K (40 layers of H=40, L_q=4096,
B=32768, plus the 16-chunk gate over 24x45x45x16 fp32 latents).

Metric: clean KV tokens scored+selected per second per head (= L_k / step
time, summed over ranks); the gate's GB/s and each kernel's roofline fraction
ride along.  Multi-GPU (timing is the max over ranks, no data-path collective):
  --shard layers (default)  every rank runs an independent layer (weak scaling);
  --shard heads             one layer's heads, and the gate's chunks, are split
                            over the ranks (strong scaling: every head and every
                            chunk is independent, so nothing is exchanged).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                    [--workload NAME] [--shard layers|heads] [--heads N]
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "clean KV tokens scored+selected/s per head; L1-gate GB/s; % of roofline"
UNIT = "tokens/s/head"
FLUSH_BYTES = 256 << 20  # > 126 MB L2
# Exponentials per SM clock of a B200 probe mixing the special-function unit
# and an FMA-pipe polynomial 5:3, with nothing else running: the exp ceiling
# the importance epilogue is measured against.
EXP_PROBE_PER_CLK = 20.6


def _sms(dev):
    return torch.cuda.get_device_properties(dev).multi_processor_count


def flush_l2(buf, sink):
    """Evict every cached line: write a buffer larger than L2, then read it
    back so the dirty lines are written back now and the next timed kernel
    starts with a clean L2 (no write-back traffic of ours lands on it)."""
    buf.zero_()
    torch.sum(buf.view(torch.float32), dim=0, out=sink)


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="long_history")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first N heads of the layer (0 = all); for small "
                         "profiler captures")
    ap.add_argument("--shard", default="layers", choices=["layers", "heads"])
    ap.add_argument("--serial", action="store_true",
                    help="run the five calls one after another on one stream")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the timings of the cache commit, mask consumer and history gate")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the full step of the full-step sweep (40 layers at L_k=128K)")
    ap.add_argument("--sweep-lk", default="131072",
                    help="comma-separated L_k values of the full-step sweep to time "
                         "(of 4096, 16384, 65536, 131072)")
    ap.add_argument("--ref-frac", type=int, default=16,
                    help="the oracle legs time 1/N of a head's importance rows and a 1/N key "
                         "subset of its redundancy per sampled head")
    return ap.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """SM clocks and clock-event (throttle) reasons sampled during timing.

    NVML is polled from a background thread every ~2 ms (only reads: nothing
    about the GPU is changed); without NVML, nvidia-smi is polled every 100 ms.
    The device is found by its PCI bus id, so that a remapped
    CUDA_VISIBLE_DEVICES still samples the GPU the rank runs on."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        p = torch.cuda.get_device_properties(device)
        self.bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        self.proc = None
        self.thread = None
        self.samples = []
        self.path = f"/tmp/fc_clocks_{os.getpid()}.csv"

    def _nvml_loop(self, nv, handle, bits):
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((mhz, [n for n, bit in bits if reasons & bit]))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        self.samples = []
        self.stop_flag = False
        try:
            import threading

            import pynvml as nv
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByPciBusId(self.bus)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            bits = [("hw_slowdown", nv.nvmlClocksEventReasonHwSlowdown),
                    ("hw_thermal_slowdown", nv.nvmlClocksEventReasonHwThermalSlowdown),
                    ("sw_thermal_slowdown", nv.nvmlClocksEventReasonSwThermalSlowdown),
                    ("sw_power_cap", nv.nvmlClocksEventReasonSwPowerCap),
                    ("hw_power_brake", nv.nvmlClocksEventReasonHwPowerBrakeSlowdown)]
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, handle, bits),
                                           daemon=True)
            self.thread.start()
            time.sleep(0.01)
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.bus, "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            return self._summary([m for m, _ in self.samples], self.max_mhz,
                                 sorted({r for _, rs in self.samples for r in rs}), "nvml")
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock sampler"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)
        reasons = sorted({self.NAMES[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return self._summary(mhz, mx, reasons, "nvidia-smi")

    @staticmethod
    def _summary(mhz, mx, reasons, source):
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"],
                    "source": source}
        loaded = [m for m in mhz if mx and m > 0.5 * mx] or mhz
        return {"sm_mhz": statistics.median(loaded), "sm_min_mhz": min(mhz), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(mhz), "source": source}


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------
def configs(workload):
    """(KV workload, gate workload or None) of a bench workload name: the
    full-step sweep layers share the 16-chunk gate; the long-history layer
    has no gate."""
    from cache_gating_kv_b200 import workloads as W

    kv_cfg = W.KV_CONFIGS[workload]
    if workload in W.GATE_CONFIGS:
        return kv_cfg, W.GATE_CONFIGS[workload]
    if workload.startswith("sweep_lk"):
        return kv_cfg, W.GATE_CONFIGS["full_step_sweep"]
    return kv_cfg, None


def workload_desc(workload):
    """The workload's name and sizes, as both arms report them."""
    kv_cfg, gate_cfg = configs(workload)
    lam = kv_cfg.lam[len(kv_cfg.lam) // 2]
    return (f"{workload}: H={kv_cfg.H} d={kv_cfg.d} L_q={kv_cfg.Lq} L_k={kv_cfg.Lk} "
            f"B={kv_cfg.B} lambda={lam} pool={kv_cfg.pool}; " +
            (f"gate {gate_cfg.n_chunks}x{gate_cfg.N} fp32 m={gate_cfg.m} eps={gate_cfg.eps[0]}"
             if gate_cfg else "no gate"))


def bench_config(workload, per_rank="one independent layer per GPU"):
    """The ``config`` object of the JSON line; both arms report the same one."""
    return {"workload": workload_desc(workload), "per_rank": per_rank,
            "l2": "flushed between steps (256 MiB write + read-back, outside the timed events)"}


# DRAM bytes (read + write) of one fc_kv_importance call over a workload's
# heads, from one ncu capture of its launches (dram__bytes_read.sum +
# dram__bytes_write.sum): workload -> (bytes per call, heads in the call).  The
# bytes per head depend on how many heads' keys are in flight at once (4 heads
# read Q and K exactly once per pass, 12 and 40 heads 1.17-1.24x in the row
# pass), so the figure holds only for the head count it was taken at; any
# other count reports null.  A change to the importance kernels voids it.
IMP_TRAFFIC = {
    # all 40 heads captured at once (the three metrics take one ncu pass):
    # row pass 1662.2 + 12.9 MB, column pass 1438.9 + 20.4 MB
    "long_history": (3134.4e6, 40),
}


def _traffic(workload, H):
    t = IMP_TRAFFIC.get(workload)
    return t[0] if t is not None and t[1] == H else None


class Step:
    """Device buffers of one step and the five C-ABI calls.  ``heads`` and
    ``chunks`` ([lo, hi) ranges) select this rank's share of the layer's heads
    and of the gate's chunks; by default the whole layer."""

    def __init__(self, kv_cfg, gate_cfg, seed, dev, heads=None, chunks=None, layer=0):
        import cache_gating_kv_b200 as fc
        from cache_gating_kv_b200 import workloads as W

        self.fc = fc
        self.kv, self.gc = kv_cfg, gate_cfg
        q, k, v = W.kv_inputs(kv_cfg, seed=seed, layer=layer,
                              heads=None if heads is None else range(*heads))
        self.host = {"q": q, "k": k, "v": v}
        n_c = 0
        if gate_cfg is not None:
            x = W.gate_initial(gate_cfg, seed)
            vel = W.gate_velocity(gate_cfg, seed)
            gstep = gate_cfg.m + 5 + gate_cfg.stagger * (gate_cfg.n_chunks - 1)
            st = W.gate_step_counters(gate_cfg, min(gstep, gate_cfg.T - 1))
            dt = W.gate_dt(gate_cfg, st)
            lo, hi = (0, gate_cfg.n_chunks) if chunks is None else chunks
            n_c = hi - lo
            if n_c > 0:
                self.host.update(x=torch.from_numpy(x[lo:hi].copy()),
                                 vel=torch.from_numpy(vel[lo:hi].copy()),
                                 dt=torch.from_numpy(dt[lo:hi].copy()),
                                 step=torch.from_numpy(st[lo:hi].copy()), f=torch.zeros(n_c))
        self.n_c = n_c
        self.d = {n: t.to(dev) for n, t in self.host.items()}
        H = q.shape[0]
        self.H = H
        Lq, Lk, d, B = kv_cfg.Lq, kv_cfg.Lk, kv_cfg.d, kv_cfg.B
        code = fc.FC_BF16 if kv_cfg.dtype == "bf16" else fc.FC_F32
        self.eps = gate_cfg.eps[0] if gate_cfg is not None else None
        self.lam = kv_cfg.lam[len(kv_cfg.lam) // 2]
        self.out = {
            "l1": torch.zeros(max(n_c, 1), device=dev),
            "mask": torch.zeros(max(n_c, 1), dtype=torch.uint8, device=dev),
            "imp": torch.empty(H, Lk, device=dev), "red": torch.empty(H, Lk, device=dev),
            "idx": torch.empty(H, B, dtype=torch.int32, device=dev),
            "ko": torch.empty(H, B, d, dtype=q.dtype, device=dev),
            "vo": torch.empty(H, B, d, dtype=q.dtype, device=dev),
        }
        self.fork = torch.cuda.Event()
        self.join = torch.cuda.Event()
        self.ws = {
            "gate": fc.workspace(fc.fc_gate_workspace_size(n_c, gate_cfg.N) if n_c else 256, dev),
            "imp": fc.workspace(fc.fc_importance_workspace_size(code, H, Lq, Lk, d), dev),
            "red": fc.workspace(fc.fc_redundancy_workspace_size(code, H, Lk, d), dev),
            "topb": fc.workspace(fc.fc_score_topb_workspace_size(H, Lk, B), dev),
        }

    # events bracketing the calls: call -> (start event, end event)
    SPANS = {"gate": ("gate0", "gate1"), "redundancy": ("gate1", "red1"),
             "importance": ("imp0", "imp1"), "score_topb": ("join", "score1"),
             "compact": ("score1", "end")}
    EVENTS = ("start", "gate0", "gate1", "red1", "imp0", "imp1", "join", "score1", "end")

    def run(self, stream, ev=None, side=None, side_after=(), compact_after=()):
        """Enqueue one step; returns the number of kernel launches the library
        enqueued.  The gate and the redundancy depend on nothing else in the
        step, so with a ``side`` stream they run there, beside the importance
        on ``stream``, and the score waits for both.  ``ev`` maps the names in
        EVENTS to timing events.  ``side_after`` / ``compact_after``: events the
        gate / the compaction must wait for (inputs still being copied in)."""
        fc, d, o, w = self.fc, self.d, self.out, self.ws
        rec = (lambda k, st: ev[k].record(st)) if ev else (lambda k, st: None)
        s2 = side if side is not None else stream
        n = 0
        rec("start", stream)
        if side is not None:
            self.fork.record(stream)
            side.wait_event(self.fork)
        for e in side_after:
            s2.wait_event(e)
        rec("gate0", s2)
        if self.n_c:
            fc.fc_chunk_l1_gate(d["x"], d["vel"], d["dt"], d["step"], self.gc.m, self.eps,
                                d["f"], o["l1"], o["mask"], w["gate"], stream=s2)
            n += fc.fc_last_launches()
        rec("gate1", s2)
        fc.fc_kv_redundancy(d["k"], o["red"], w["red"], stream=s2)
        n += fc.fc_last_launches()
        rec("red1", s2)
        rec("imp0", stream)
        fc.fc_kv_importance(d["q"], d["k"], o["imp"], w["imp"], stream=stream)
        n += fc.fc_last_launches()
        rec("imp1", stream)
        if side is not None:
            self.join.record(side)
            stream.wait_event(self.join)
        rec("join", stream)
        fc.fc_kv_score_topb(o["imp"], o["red"], self.kv.pool, self.lam, self.kv.B, o["idx"],
                            w["topb"], stream=stream)
        n += fc.fc_last_launches()
        rec("score1", stream)
        for e in compact_after:
            stream.wait_event(e)
        fc.fc_kv_compact(d["k"], d["v"], o["idx"], o["ko"], o["vo"], stream=stream)
        n += fc.fc_last_launches()
        rec("end", stream)
        return n

    def reset_gate(self):
        if self.n_c:
            self.d["x"].copy_(self.host["x"])
            self.d["f"].zero_()


def reduce_max(values, world, device):
    """Element-wise max over ranks of a few host floats (identity at world 1)."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def shard_heads(H, rank, world):
    """Contiguous head range [lo, hi) of `rank` when one layer's heads are split
    over `world` GPUs (every head is independent: no exchange is needed)."""
    per, extra = divmod(H, world)
    lo = rank * per + min(rank, extra)
    return lo, lo + per + (1 if rank < extra else 0)


def _bytes_gate(gc):
    return 12 * gc.n_chunks * gc.N


def native(a, rank, world, local_rank):
    from cache_gating_kv_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    kv_cfg, gate_cfg = configs(a.workload)
    by_heads = a.shard == "heads" and world > 1
    if by_heads:
        if world > kv_cfg.H:
            raise SystemExit(f"--shard heads needs at most H={kv_cfg.H} ranks")
        heads = shard_heads(kv_cfg.H, rank, world)
        chunks = shard_heads(gate_cfg.n_chunks, rank, world) if gate_cfg else None
        step = Step(kv_cfg, gate_cfg, seed=0, dev=dev, heads=heads, chunks=chunks)
        per_rank = (f"heads [{heads[0]}, {heads[1]}) of one layer"
                    + (f", gate chunks [{chunks[0]}, {chunks[1]})" if chunks else ""))
    elif a.heads > 0:
        step = Step(kv_cfg, gate_cfg, seed=rank, dev=dev, heads=(0, min(a.heads, kv_cfg.H)))
        per_rank = f"the first {min(a.heads, kv_cfg.H)} heads of one layer per GPU"
    else:
        step = Step(kv_cfg, gate_cfg, seed=rank, dev=dev)
        per_rank = "one independent layer per GPU"
    # the importance (on the critical path) gets the higher priority; the gate
    # and the redundancy fill the SMs it leaves idle
    lo, hi = torch.cuda.Stream.priority_range()
    stream = torch.cuda.Stream(device=dev, priority=hi)
    side = None if a.serial else torch.cuda.Stream(device=dev, priority=lo)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    names = list(Step.SPANS)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def events(external):
        return {k: torch.cuda.Event(enable_timing=True, external=external) for k in Step.EVENTS}

    # One step is captured once as a CUDA graph (with timing events as graph
    # nodes) and replayed: the GPU runs the step's launches back to back
    # instead of waiting on the host between small kernels.
    ev = events(True)
    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            flush_l2(flush, sink)
            step.run(stream, side=side)
        torch.cuda.synchronize()
        eager_ev = events(False)
        flush_l2(flush, sink)
        launches_per_step = step.run(stream, eager_ev, side=side)
        torch.cuda.synchronize()
        ms_eager = eager_ev["start"].elapsed_time(eager_ev["end"])
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="relaxed"):
            step.run(stream, ev, side=side)
        for _ in range(2):
            flush_l2(flush, sink)
            graph.replay()
        torch.cuda.synchronize()
        clocks = Clocks(dev)
        barrier()
        torch.cuda.synchronize()
        clocks.start()
        per = {n: [] for n in names}
        tot = []
        for i in range(a.steps):
            flush_l2(flush, sink)  # between steps, outside the timed events
            graph.replay()
            stream.synchronize()
            for n, (e0, e1) in Step.SPANS.items():
                per[n].append(ev[e0].elapsed_time(ev[e1]))
            tot.append(ev["start"].elapsed_time(ev["end"]))
        torch.cuda.synchronize()
        barrier()
        ck = clocks.stop()
        # each call alone (one stream, one after another) for its own roofline
        alone = per
        if side is not None:
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1, stream=stream, capture_error_mode="relaxed"):
                step.run(stream, ev)
            alone = {n: [] for n in names}
            for i in range(a.steps + 2):
                flush_l2(flush, sink)
                g1.replay()
                stream.synchronize()
                if i >= 2:
                    for n, (e0, e1) in Step.SPANS.items():
                        alone[n].append(ev[e0].elapsed_time(ev[e1]))
            del g1
        gates = {}
        for gname in ("bf16_layer", "bf16_large_head", "full_step_sweep"):
            gc = W.GATE_CONFIGS[gname]
            ms_g = _gate_alone(gc, rank, dev, stream, flush, sink, max(a.steps, 10))
            gb = _bytes_gate(gc) / (ms_g * 1e-3) / 1e9
            gates[gname] = {"chunks": gc.n_chunks, "n_per_chunk": gc.N, "us": ms_g * 1e3,
                            "GB/s": gb, "frac_hbm": gb / _peaks()[0]}
        nxt = None
        if not a.no_next:
            hbm0, tf0, _, _ = _peaks()
            nxt = _next_rows(step, dev, stream, flush, sink, max(3, min(a.steps, 10)), hbm0, tf0)
        sweep = None
        if not a.no_sweep:
            sweep = {}
            for lk in (int(x) for x in a.sweep_lk.split(",")):
                sweep[f"L_k={lk}"] = _full_step_sweep(dev, stream, side, flush, sink, rank, lk)
        barrier()
    del graph
    ms_step = sum(tot) / len(tot)
    ms_call = {n: sum(v) / len(v) for n, v in per.items()}
    ms_alone = {n: sum(v) / len(v) for n, v in alone.items()}

    # end to end through the public API with host buffers (pinned), every step
    e2e = None
    if not a.no_e2e:
        e2e = _e2e(step, stream, side, flush, sink, a, dev)

    maxed = reduce_max([ms_step] + ([e2e["ms"]] if e2e else []), world, dev)
    t_max = maxed[0]
    if e2e:
        e2e["ms"] = maxed[1]
    H, Lq, Lk, d = step.H, kv_cfg.Lq, kv_cfg.Lk, kv_cfg.d
    # tokens/s per head over all ranks: each rank finishes a layer per step (by
    # layers), or all ranks together finish one layer per step (by heads)
    layers = 1 if by_heads else world
    value = layers * Lk / (t_max * 1e-3)
    hbm, tf_burst, tf_sus, src = _peaks()
    # The denominator for the importance: the burst GEMM figure, or the
    # sustained one when the timed steps ran under the power cap (the regime
    # in which that figure was measured: a GEMM loop held for seconds).
    capped = "sw_power_cap" in (ck.get("reasons") or [])
    tf_peak = tf_sus if capped else tf_burst
    exec_flops = 4.0 * H * Lq * Lk * d  # two passes of Q K^T
    imp_tf = exec_flops / (ms_call["importance"] * 1e-3) / 1e12
    gexp = 2.0 * H * Lq * Lk / (ms_call["importance"] * 1e-3) / 1e9
    gate_gbs = (_bytes_gate(gate_cfg) * step.n_c / gate_cfg.n_chunks / (ms_alone["gate"] * 1e-3)
                / 1e9) if step.n_c else None
    elem = 2 if kv_cfg.dtype == "bf16" else 4
    red_gbs = H * Lk * d * elem / (ms_alone["redundancy"] * 1e-3) / 1e9
    comp_gbs = 2 * 2 * H * kv_cfg.B * d * elem / (ms_alone["compact"] * 1e-3) / 1e9
    topb_gbs = (H * Lk * 8 + H * kv_cfg.B * 4) / (ms_alone["score_topb"] * 1e-3) / 1e9
    launches = launches_per_step * a.steps
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": t_max, "higher_is_better": True,
        "scaling": "strong" if by_heads else "weak",
        "vs_baseline": None, "dtype": kv_cfg.dtype if kv_cfg.dtype == "bf16" else "f32",
        "data": "synthetic (seeded AR(1) keys, N(0,1) queries/values, flow-matching toy latents)",
        "config": bench_config(a.workload, per_rank),
        "roofline": {"bound": "tensor", "kernel": "fc_kv_importance (2 passes)",
                     # achieved: the method's flops (one Q K^T per call, 2*H*Lq*Lk*d);
                     # the two passes execute twice that (frac_executed)
                     "achieved": imp_tf / 2, "peak": tf_peak, "unit": "TFLOP/s",
                     "frac": imp_tf / 2 / tf_peak,
                     "peak_source": f"{src} bf16 " + (
                         "sustained (the timed steps ran under sw_power_cap)" if capped
                         else "burst"),
                     "flops_per_launch": exec_flops / 2,
                     "executed_flops_per_launch": exec_flops,
                     "frac_executed": imp_tf / tf_peak,
                     "frac_of_burst_peak": imp_tf / 2 / tf_burst,
                     "frac_of_sustained_peak": imp_tf / 2 / tf_sus,
                     "traffic": _traffic(a.workload, H),
                     "traffic_unit": "bytes per call (DRAM read + write of the call's "
                                     "launches, from one ncu capture of this workload)"},
        "kernels_ms": ms_call,
        "kernels_ms_alone": ms_alone,
        "kernels_note": "kernels_ms: spans inside the timed step (gate and redundancy share "
                        "the GPU with the importance there); kernels_ms_alone: the same calls "
                        "one after another on one stream, which the GB/s figures use",
        "gate": {"GB/s": gate_gbs, "frac_hbm": gate_gbs / hbm if gate_gbs else None},
        "next_rows": nxt,
        "gate_workloads": dict(gates, note="each gate step alone, CUDA graph, L2 flushed "
                               "before every replay; 12 B moved per latent element"),
        "timing": "one step captured as a CUDA graph, replayed per step; CUDA events are "
                  "graph nodes around each call" +
                  ("" if a.serial else "; gate and redundancy on a second, lower-priority "
                   "stream beside the importance (they depend on nothing else in the step)") +
                  f"; eager (host-launched) step for reference: {ms_eager:.3f} ms",
        "importance": {"TFLOP/s executed": imp_tf, "TFLOP/s algorithmic": imp_tf / 2,
                       "Gexp/s": gexp,
                       "frac_of_exp_probe": gexp * 1e9 / (EXP_PROBE_PER_CLK * _sms(dev) *
                                                         (ck.get("sm_mhz") or 1965) * 1e6),
                       "note": "both passes recompute Q K^T (executed = 2 x algorithmic "
                               "flops); 2 exponentials per score; frac_of_exp_probe: against "
                               f"{EXP_PROBE_PER_CLK} exps/clock/SM at the sampled SM clock"},
        "redundancy": {"GB/s": red_gbs, "frac_hbm": red_gbs / hbm},
        "score_topb": {"GB/s": topb_gbs, "frac_hbm": topb_gbs / hbm,
                       "bytes": "8 B read per token (imp, red) + 4 B written per kept index"},
        "compact": {"GB/s": comp_gbs, "frac_hbm": comp_gbs / hbm},
        "gpu_launches": launches,
        "clocks": ck,
    }
    if sweep is not None:
        out["full_step_sweep"] = sweep
    if e2e:
        out["e2e"] = {"value": layers * Lk / (e2e["ms"] * 1e-3), "unit": UNIT,
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]}
    return out


def _graph_ms(fn, stream, flush, sink, steps, warm=3):
    """Mean CUDA-graph-timed duration (ms) of ``fn`` enqueued on ``stream``,
    with L2 flushed before every replay."""
    with torch.cuda.stream(stream):
        fn()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            e0.record(stream)
            fn()
            e1.record(stream)
        times = []
        for i in range(steps + warm):
            flush_l2(flush, sink)
            g.replay()
            stream.synchronize()
            if i >= warm:
                times.append(e0.elapsed_time(e1))
        del g
    return sum(times) / len(times)


def _next_rows(step, dev, stream, flush, sink, steps, hbm, tf_peak):
    """The rows built beyond the per-step path, each timed alone: the mask
    consumer and the history-guided gate on the 16-chunk full-step-sweep
    latents, and one cache commit that compresses a full one-layer buffer."""
    import cache_gating_kv_b200 as fc
    from cache_gating_kv_b200 import workloads as W

    gc = W.GATE_CONFIGS["full_step_sweep"]
    n_c, N = gc.n_chunks, gc.N
    x = torch.from_numpy(W.gate_initial(gc, 0)).to(dev)
    v = torch.from_numpy(W.gate_velocity(gc, 0)).to(dev)
    mask = torch.zeros(n_c, dtype=torch.uint8, device=dev)
    mask[::2] = 1  # half the chunks recompute
    n_re = int(mask.sum().item())
    dense = torch.empty_like(x)
    ids = torch.empty(n_c, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    v_cache = v.clone()
    ms_g = _graph_ms(lambda: fc.fc_gather_recompute(x, mask, dense, ids, cnt, stream=stream),
                     stream, flush, sink, steps)
    ms_s = _graph_ms(lambda: fc.fc_scatter_velocity(dense, ids, cnt, v_cache, stream=stream),
                     stream, flush, sink, steps)
    moved = 2 * n_re * N * 4
    h_new = x.clone()
    h_old = x + 0.01 * v
    st = torch.full((n_c,), gc.m + 3, dtype=torch.int32, device=dev)
    f = torch.zeros(n_c, device=dev)
    dd = torch.empty(n_c, device=dev)
    rf = torch.empty(n_c, dtype=torch.uint8, device=dev)
    ws = fc.workspace(fc.fc_gate_workspace_size(n_c, N), dev)
    ms_h = _graph_ms(lambda: fc.fc_history_l1_gate(h_old, h_new, st, gc.m, 0.05, f, dd, rf, ws,
                                                   stream=stream), stream, flush, sink, steps)
    del x, v, dense, v_cache, h_new, h_old
    # one compression of a full cache: the step's layer as the buffer, C = L_k / 4
    kv = step.kv
    H, Lq, Lk, d = step.H, kv.Lq, kv.Lk, kv.d
    C, Bb = Lk // 4, Lk - Lk // 4
    qd, kb, vb = step.d["q"], step.d["k"], step.d["v"]
    kn, vn = torch.empty_like(kb), torch.empty_like(vb)
    code = fc.FC_BF16 if kb.dtype == torch.bfloat16 else fc.FC_F32
    cws = fc.workspace(fc.fc_kv_cache_workspace_size(code, H, Lq, Bb, C, d), dev)
    ms_c = _graph_ms(lambda: fc.fc_kv_cache_commit(qd, kb, vb, kn, vn, Bb, C, cws, kv.pool,
                                                   0.5, stream=stream),
                     stream, flush, sink, steps)
    imp_flops = 4.0 * H * Lq * Lk * d
    return {
        "gather_recompute": {"us": ms_g * 1e3, "GB/s": moved / (ms_g * 1e-3) / 1e9,
                             "frac_hbm": moved / (ms_g * 1e-3) / 1e9 / hbm,
                             "workload": f"{n_re} of {n_c} chunks x {N} fp32"},
        "scatter_velocity": {"us": ms_s * 1e3, "GB/s": moved / (ms_s * 1e-3) / 1e9,
                             "frac_hbm": moved / (ms_s * 1e-3) / 1e9 / hbm,
                             "workload": f"{n_re} of {n_c} chunks x {N} fp32"},
        "history_gate": {"us": ms_h * 1e3, "GB/s": _bytes_gate(gc) / (ms_h * 1e-3) / 1e9,
                         "frac_hbm": _bytes_gate(gc) / (ms_h * 1e-3) / 1e9 / hbm,
                         "workload": f"{n_c} segments x {N} fp32"},
        "cache_commit": {"ms": ms_c, "TFLOP/s importance-executed per commit":
                         imp_flops / (ms_c * 1e-3) / 1e12,
                         "frac_bf16": imp_flops / (ms_c * 1e-3) / 1e12 / tf_peak,
                         "workload": f"H={H} d={d} L_q={Lq} C={C} B_budget={Bb} (a full "
                                     f"buffer of B_budget + C candidates, {kv.dtype})"},
    }


def _full_step_sweep(dev, stream, side, flush, sink, seed, lk=131072, layers=40, steps=2,
                     warm=1):
    """The full step of the full-step sweep at one L_k: ``layers`` layers of
    H=40, L_q=4096, B=L_k/4 through importance, redundancy, score/top-B and
    compaction, plus one gate step over the 16 chunks, timed with CUDA events
    on the launching stream (L2 flushed between steps).  The layers alternate
    between two seeded layers' inputs (drawing 40 distinct layers on the host
    would take minutes); at L_k = 131072 each layer's K and V are 1.34 GB
    apiece, ten times the L2, so no layer finds the previous one's data in
    cache (at L_k = 4096 a layer's K is 42 MB, and the alternation keeps the
    two layers apart by one layer's traffic)."""
    import cache_gating_kv_b200 as fc
    from cache_gating_kv_b200 import workloads as W

    kv, gc = W.KV_CONFIGS[f"sweep_lk{lk}"], W.GATE_CONFIGS["full_step_sweep"]
    ls = [Step(kv, None, seed=seed, dev=dev, layer=i) for i in range(2)]
    g = _gate_bufs(gc, seed, dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)

    def one():
        ev0.record(stream)
        fork = torch.cuda.Event()
        fork.record(stream)
        s2 = side if side is not None else stream
        s2.wait_event(fork)
        fc.fc_chunk_l1_gate(g["x"], g["v"], g["dt"], g["st"], gc.m, gc.eps[0], g["f"], g["l1"],
                            g["mask"], g["ws"], stream=s2)
        for i in range(layers):
            ls[i % 2].run(stream, side=side)
        ev1.record(stream)

    times = []
    with torch.cuda.stream(stream):
        for i in range(warm + steps):
            flush_l2(flush, sink)
            g["f"].zero_()
            torch.cuda.synchronize()
            one()
            torch.cuda.synchronize()
            if i >= warm:
                times.append(ev0.elapsed_time(ev1))
    ms = sum(times) / len(times)
    H, Lq, Lk, d = kv.H, kv.Lq, kv.Lk, kv.d
    del ls, g
    return {"workload": f"{layers} layers x sweep_lk{lk} (H={H} d={d} L_q={Lq} L_k={Lk} "
                        f"B={kv.B} bf16) + gate {gc.n_chunks}x{gc.N} fp32",
            "ms_per_step": ms, "steps": steps,
            "tokens/s/head": layers * Lk / (ms * 1e-3),
            "TFLOP/s importance-executed over the step": layers * 4.0 * H * Lq * Lk * d /
            (ms * 1e-3) / 1e12,
            "inputs": "two seeded layers' inputs, alternating over the 40 layers",
            "timing": "CUDA events on the launching stream around the whole step (eager "
                      "launches); the gate and each layer's redundancy on the side stream"}


def _gate_bufs(gc, seed, dev):
    """Device buffers of one gate step over every chunk of ``gc`` (every chunk
    active, past its forced steps)."""
    import cache_gating_kv_b200 as fc
    from cache_gating_kv_b200 import workloads as W

    n = gc.n_chunks
    return {"x": torch.from_numpy(W.gate_initial(gc, seed)).to(dev),
            "v": torch.from_numpy(W.gate_velocity(gc, seed)).to(dev),
            "st": torch.full((n,), gc.m + 3, dtype=torch.int32, device=dev),
            "dt": torch.full((n,), 0.001, device=dev), "f": torch.zeros(n, device=dev),
            "l1": torch.zeros(n, device=dev),
            "mask": torch.zeros(n, dtype=torch.uint8, device=dev),
            "ws": fc.workspace(fc.fc_gate_workspace_size(n, gc.N), dev)}


def _gate_alone(gc, seed, dev, stream, flush, sink, steps):
    """Gate step over every chunk of ``gc`` alone, CUDA-graph timed (ms)."""
    import cache_gating_kv_b200 as fc

    b = _gate_bufs(gc, seed, dev)
    x, v, st, dt, f, l1, mask, ws = (b[k] for k in ("x", "v", "st", "dt", "f", "l1", "mask",
                                                    "ws"))
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    fc.fc_chunk_l1_gate(x, v, dt, st, gc.m, gc.eps[0], f, l1, mask, ws, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        e0.record(stream)
        fc.fc_chunk_l1_gate(x, v, dt, st, gc.m, gc.eps[0], f, l1, mask, ws, stream=stream)
        e1.record(stream)
    times = []
    for i in range(steps + 3):
        flush_l2(flush, sink)
        g.replay()
        stream.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    del g
    return sum(times) / len(times)


def _e2e(step, stream, side, flush, sink, a, dev):
    """Same step with pinned host inputs copied in and the results read back,
    inside the timed region, every step."""
    host_in = {n: t.pin_memory() for n, t in step.host.items()}
    res = (["l1", "mask"] if step.n_c else []) + ["idx"]
    host_out = {n: torch.empty_like(step.out[n], device="cpu").pin_memory() for n in res}
    if step.n_c:
        res.append("f")
        host_out["f"] = torch.empty_like(step.host["f"]).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    # With a side stream the copies are ordered for overlap: Q and K first (the
    # importance and the redundancy need them), then the gate's inputs and V on
    # a copy stream while the importance runs; the gate waits for its inputs,
    # the compaction for V.  The PCIe link carries one copy after another.
    first = [n for n in ("q", "k") if n in host_in]
    later = [n for n in host_in if n not in first and n != "v"] + ["v"]
    cp = torch.cuda.Stream(device=dev) if side is not None else None
    times = []
    with torch.cuda.stream(stream):
        for i in range(a.warmup + a.steps):
            flush_l2(flush, sink)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if cp is None:
                for n, t in host_in.items():
                    step.d[n].copy_(t, non_blocking=True)
                step.run(stream)
            else:
                for n in first:
                    step.d[n].copy_(host_in[n], non_blocking=True)
                qk = torch.cuda.Event()
                qk.record(stream)
                cp.wait_event(qk)
                with torch.cuda.stream(cp):
                    for n in later[:-1]:
                        step.d[n].copy_(host_in[n], non_blocking=True)
                    gate_in = torch.cuda.Event()
                    gate_in.record(cp)
                    step.d["v"].copy_(host_in["v"], non_blocking=True)
                    v_in = torch.cuda.Event()
                    v_in.record(cp)
                step.run(stream, side=side, side_after=(gate_in,), compact_after=(v_in,))
            for n in res:
                host_out[n].copy_(step.d["f"] if n == "f" else step.out[n], non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if i >= a.warmup:
                times.append(e0.elapsed_time(e1))
    return {"ms": sum(times) / len(times), "h2d": h2d, "d2h": d2h}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------
def _oracle_sample(kv_cfg, gate_cfg, head, frac, seed=0):
    """Times the oracle, as it stands, on a bounded sample of one step and
    returns ``(measured seconds, estimated seconds of the whole step)``.

    The sample is one head of the layer: the importance over its first
    L_q/frac query rows (every key; the rows are independent, so the head's
    time is that x frac), the redundancy of its first L_k/frac keys (the
    brute-force cosine matrix is L_k^2 work, so the head's time is estimated
    as that x frac^2), the score/top-B and the compaction of the whole head, and
    one full gate step (when the workload has one).  Step estimate = gate +
    H x the head's estimate."""
    from cache_gating_kv_b200 import workloads as W
    from oracle import flowcache_oracle as O

    q, k, v = W.kv_inputs(kv_cfg, seed=seed, heads=[head % kv_cfg.H])
    nq = max(1, kv_cfg.Lq // frac)
    nr = max(2, kv_cfg.Lk // frac)
    q64 = q[:, :nq].float().numpy().astype(np.float64)
    k64 = k.float().numpy().astype(np.float64)
    kf, vf = k.float().numpy(), v.float().numpy()
    lam = kv_cfg.lam[len(kv_cfg.lam) // 2]
    t_gate = 0.0
    if gate_cfg is not None:
        x = W.gate_initial(gate_cfg, seed)
        vel = W.gate_velocity(gate_cfg, seed)
        st = W.gate_step_counters(gate_cfg, gate_cfg.m + 5)
        dt = W.gate_dt(gate_cfg, st)
        t0 = time.perf_counter()
        O.gate_step(x, vel, dt, st, gate_cfg.m, gate_cfg.eps[0],
                    np.zeros(gate_cfg.n_chunks, np.float32))
        t_gate = time.perf_counter() - t0
    t0 = time.perf_counter()
    imp = O.importance(q64, k64)
    t_imp = time.perf_counter() - t0
    t0 = time.perf_counter()
    red = O.redundancy(k64[:, :nr])
    t_red = time.perf_counter() - t0
    red_full = np.resize(red, (1, kv_cfg.Lk))  # a full-length vector for the selection's timing
    t0 = time.perf_counter()
    _, idx = O.score_topb(imp, red_full, lam, kv_cfg.pool, kv_cfg.B)
    O.compact(kf, vf, idx)
    t_rest = time.perf_counter() - t0
    measured = t_gate + t_imp + t_red + t_rest
    head_est = t_imp * (kv_cfg.Lq / nq) + t_red * (kv_cfg.Lk / nr) ** 2 + t_rest
    return measured, t_gate + kv_cfg.H * head_est


def _sample_desc(kv_cfg, frac):
    return (f"one head per sample: the importance of its first {max(1, kv_cfg.Lq // frac)} of "
            f"{kv_cfg.Lq} query rows (x{frac}), the redundancy of its first "
            f"{max(2, kv_cfg.Lk // frac)} of {kv_cfg.Lk} keys (x{frac}^2, quadratic work), the "
            f"score/top-B and compaction of the whole head, plus one full gate step when the "
            f"workload has one; step estimate = gate + H x head estimate")


def _cores():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(a, samples=4):
    kv_cfg, gate_cfg = configs(a.workload)
    est = [_oracle_sample(kv_cfg, gate_cfg, h, a.ref_frac)[1] for h in range(samples)]
    t_step = sum(est) / len(est)
    return {"value": kv_cfg.Lk / t_step, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"{samples} samples; " + _sample_desc(kv_cfg, a.ref_frac),
            "est_ms_per_step": t_step * 1e3}


def reference(a, rank):
    """The reference arm: the oracle on the host cores, on this arm's workload,
    metric and unit.  Each step times one bounded sample (`_oracle_sample`);
    ``ms_per_step`` is the time measured per step, and the value is L_k over
    the estimated time of a whole step."""
    if rank != 0:
        return None
    kv_cfg, gate_cfg = configs(a.workload)
    meas, est = [], []
    for i in range(a.warmup + a.steps):
        m, e = _oracle_sample(kv_cfg, gate_cfg, i, a.ref_frac, seed=0)
        if i >= a.warmup:
            meas.append(m)
            est.append(e)
    t_est = sum(est) / len(est)
    value = kv_cfg.Lk / t_est
    sample = _sample_desc(kv_cfg, a.ref_frac)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": sum(meas) / len(meas) * 1e3,
            "est_ms_per_full_step": t_est * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": bench_config(a.workload),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "note": "ms_per_step is the time each step's sample took; value = L_k / "
                    "est_ms_per_full_step, the sample scaled to a whole step"}


def main():
    a = _args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if a.impl == "reference":
        out = reference(a, rank)
        if out is not None:
            print(json.dumps(out))
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = native(a, rank, world, local_rank)
        if rank == 0:
            if not a.no_cpu_baseline and world == 1:  # the oracle's baseline: rank 0 at N=1
                out["cpu_baseline"] = cpu_baseline(a)
            print(json.dumps(out))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
