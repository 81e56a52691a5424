"""Benchmark of the VideoMLA latent-KV hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input at
the Wan-1.3B layer shape: ``videomla_cache_write`` of a 3-frame chunk (4680
tokens) into slots 18-20 of a 21-slot ring, then ``videomla_attention`` of those
4680 queries over the 21-frame window (32760 keys), 12 heads.  The ring is
prefilled (untimed) by the same cache-write kernel.

Metric: TFLOP/s of the step, counted with the algorithmic flops of the absorbed
form (App. E): per (query, key, head) 2 (d_c + d_rope) + 2 d_c = 832,
plus per (query, head) 2 d_nope d_c (absorption) + 2 d_c d_v (W_uv epilogue),
plus 2 (d_c + d_rope) d_model per written token.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
N > 1 runs under torchrun, one rank per GPU, each rank an independent replica
of the workload (no collective on the data path; weak scaling).
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
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mla_latent_kv_write_b200 import inputs as I  # noqa: E402

METRIC = "latent-KV MLA attention TFLOP/s and % of B200 bf16 peak, 21-frame window"
WORKLOAD = I.WORKLOADS["wan_layer"]
N_SETS = 4  # rotating input sets: 4 x ~60 MB > 126 MB L2


def flops_attention(d: I.Dims, B: int, Nq: int, Nk: int) -> float:
    per_qkh = 2 * (d.d_c + d.d_rope) + 2 * d.d_c
    per_qh = 2 * d.d_nope * d.d_c + 2 * d.d_c * d.d_v
    return float(B * d.n_heads * (Nq * Nk * per_qkh + Nq * per_qh))


def flops_explicit_equivalent(d: I.Dims, B: int, Nq: int, Nk: int) -> float:
    # dense MHA on reconstructed keys / values: QK^T over 128 + PV over 128, plus
    # reconstruction of K_nope and V for every key and head
    dh = d.d_nope + d.d_rope
    return float(B * d.n_heads * (Nq * Nk * (2 * dh + 2 * d.d_v) + Nk * 2 * d.d_c * (d.d_nope + d.d_v)))


def flops_cache_write(d: I.Dims, B: int, n_tok: int) -> float:
    return float(2 * B * n_tok * (d.d_c + d.d_rope) * d.d_model)


def bytes_cache_write(d: I.Dims, B: int, n_tok: int) -> float:
    return float(B * n_tok * (2 * d.d_model + 2 * (d.d_c + d.d_rope)))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return m, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            t = json.load(f)
        e = t.get(kernel)
        if not e:
            return None
        import hashlib
        h = hashlib.sha256()
        for s in e["sources"]:
            with open(os.path.join(ROOT, s), "rb") as fh:
                h.update(fh.read())
        if e.get("sources_sha256") != h.hexdigest():
            return None
        return e.get("dram_bytes_per_launch")
    except Exception:
        return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of this rank's GPU while
    the timed region runs: NVML read every 2 ms from a thread (device found by
    its PCI bus id, so CUDA_VISIBLE_DEVICES cannot point it at another GPU), or
    nvidia-smi every 200 ms if NVML is unavailable.  Reads only."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                   ("sw_power_cap", 0x4))

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.rows = []
        self.thread = None
        self.stop = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.index)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            max_sm = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()

            def run():
                while not self.stop.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                        self.rows.append((sm, max_sm, pw, rs))
                    except Exception:
                        pass
                    self.stop.wait(0.002)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            self.source = "nvml, 2 ms"
        except Exception:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi, 200 ms"
            except (OSError, ValueError):
                self.proc = None
            time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        names = tuple(n for n, _ in self.REASON_BITS)
        rows = []
        if self.thread is not None:
            for sm, mx, pw, rs in self.rows:
                rows.append((sm, mx, pw, [("active" if rs & bit else "not active") for _, bit in self.REASON_BITS]))
        elif self.proc is not None and self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                    except ValueError:
                        continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(loaded), "samples_all": len(rows),
                "sm_mhz_range_all": [min(r[0] for r in rows), max(r[0] for r in rows)], "reasons": reasons,
                "source": self.source}


def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun env).  Each rank runs an independent replica
    of the workload: the process group only carries barriers and the max of the
    per-rank timings, never data of the hot path."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, cuda: bool = True):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def job_throughput(world: int, units_per_rank: float, ms_max: float, steps: int) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3 / steps)


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of query rows
# ---------------------------------------------------------------------------

def cpu_oracle_sample(target_s: float = 12.0):
    """The fp64 oracle on the host cores, on one step of the workload: the cache
    write of the whole 4680-token chunk (timed in full) and the attention of a
    bounded, evenly spaced sample of its query rows (all heads, all keys).  Query
    rows are independent, so the step time is extrapolated linearly from the
    sample: t_step = t_cache_write + t_attention_sample * n_query / n_sample."""
    from oracle import videomla_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = len(os.sched_getaffinity(0))
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    Nk = wl.slots * T_f
    seed = I.seed_for(wl.index, 0, 0)
    w = I.layer_weights(d, seed)
    f = I.to_numpy64
    x = f(I.tokens(d, wl.batch, wl.n_query, seed + 3))
    ring = np.zeros((wl.batch, Nk, d.cache_width))
    t0 = time.perf_counter()
    O.cache_write(x, f(w["W_dkv"]), f(w["W_kr"]), f(w["gamma"]), d.rms_eps, ring, wl.slots, wl.prefill, T_f)
    t_cw = time.perf_counter() - t0
    q = I.queries(d, wl.batch, wl.n_query, seed + 1)
    cache = I.latent_cache(d, wl.batch, wl.slots, seed + 2)
    args = (f(q["q_nope"]), f(q["q_rope"]), f(w["W_uk"]), f(w["W_uv"]), f(cache), wl.slots, 0, wl.slots,
            d.grid_h, d.grid_w, d.d_c, d.rope_base, d.pairs)
    rows = np.arange(16)
    t0 = time.perf_counter()
    O.attention_absorbed(*args, query_rows=rows)
    t_probe = time.perf_counter() - t0
    n = int(min(wl.n_query, max(16, 16 * max(target_s - t_cw, 1.0) / max(t_probe, 1e-3))))
    rows = np.linspace(0, wl.n_query - 1, n).astype(int)
    t0 = time.perf_counter()
    O.attention_absorbed(*args, query_rows=rows)
    t_attn = time.perf_counter() - t0
    t_step = t_cw + t_attn * wl.n_query / n
    fl_step = flops_attention(d, wl.batch, wl.n_query, Nk) + flops_cache_write(d, wl.batch, wl.n_query)
    return {"value": fl_step / t_step / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "seconds_per_step": t_step, "extrapolated": n < wl.n_query,
            "seconds_measured": t_cw + t_attn, "cache_write_seconds": t_cw, "attention_sample_seconds": t_attn,
            "query_tokens_per_s": wl.n_query / t_step,
            "sample": f"one step: cache write of all {wl.n_query} tokens (fp64, timed in full) + attention "
                      f"(absorbed fp64 form) of {n} evenly spaced of {wl.n_query} query rows, all {d.n_heads} "
                      f"heads, all {Nk} keys; step time extrapolated linearly over the query rows"}


def workload_config(world: int) -> dict:
    """The ``config`` object of the JSON line, the same for both arms."""
    wl = WORKLOAD
    d = wl.dims
    Nk = wl.slots * d.tokens_per_frame
    return {
        "workload": "wan_layer: Wan-1.3B-shaped VideoMLA layer, B=1, 12 heads, d_c=192, d_rope=32, "
                    "d_nope=96, d_v=128, 30x52 grid, cache_write of 3 frames (4680 tokens) into a "
                    "21-slot ring + attention of 4680 queries x 32760 keys",
        "global_batch": wl.batch * world, "query_tokens_per_step": wl.n_query, "keys": Nk,
        "parallelism": f"replicas x{world} (no data-path collective)",
        "l2": f"inputs larger than L2: {N_SETS} rotating input sets (~60 MB each)",
        "flops_per_step": flops_attention(d, wl.batch, wl.n_query, Nk) + flops_cache_write(d, wl.batch, wl.n_query),
    }


def run_reference(args):
    world, rank = int(os.environ.get("WORLD_SIZE", str(args.gpus))), int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals, steps_s = [], []
    base = None
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(target_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
        if i >= args.warmup:
            vals.append(r["value"])
            steps_s.append(r["seconds_per_step"])
            base = r
    v = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(steps_s) * 1e3,
        "ms_per_step_kind": "extrapolated from a bounded sample of each step (see cpu_baseline.sample)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(world),
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": base["cores"], "kind": "oracle",
                         "sample": base["sample"], "seconds_per_step": base["seconds_per_step"],
                         "seconds_measured": base["seconds_measured"], "extrapolated": base["extrapolated"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def make_sets(dev, n_sets: int):
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    sets = []
    for k in range(n_sets):
        seed = I.seed_for(wl.index, k, 0)
        w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
        prefill = I.tokens(d, wl.batch, wl.prefill * T_f, seed + 3).to(dev)
        x = I.tokens(d, wl.batch, wl.chunk * T_f, seed + 4)
        q = I.queries(d, wl.batch, wl.n_query, seed + 5)
        cache = torch.zeros(wl.batch, wl.slots * T_f, d.cache_width, dtype=torch.bfloat16, device=dev)
        V.cache_write(prefill, w["W_dkv"], w["W_kr"], w["gamma"], cache, d, wl.slots, 0)
        del prefill
        sets.append({
            "w": w, "cache": cache, "x": x.to(dev), "q_nope": q["q_nope"].to(dev), "q_rope": q["q_rope"].to(dev),
            "out": torch.empty(wl.batch, wl.n_query, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev),
            "x_host": x.pin_memory(), "q_nope_host": q["q_nope"].pin_memory(),
            "q_rope_host": q["q_rope"].pin_memory(),
            "out_host": torch.empty(wl.batch, wl.n_query, d.n_heads, d.d_v, dtype=torch.bfloat16).pin_memory(),
        })
    torch.cuda.synchronize()
    return sets


def step(s, ev=None):
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    w = s["w"]
    if ev is not None:
        ev[0].record()
    V.cache_write(s["x"], w["W_dkv"], w["W_kr"], w["gamma"], s["cache"], d, wl.slots, wl.prefill)
    if ev is not None:
        ev[1].record()
    V.attention(s["q_nope"], s["q_rope"], w["W_uk"], w["W_uv"], s["cache"], d, wl.slots, 0, wl.slots, out=s["out"])
    if ev is not None:
        ev[2].record()


def run_e2e(sets, n_steps: int):
    """``n_steps`` steps through the public API with host buffers, pipelined the
    way a server would run them: step i's inputs (x, q_nope, q_rope) go up from
    pinned memory on a copy stream while step i-1 computes, step i's output
    comes back on a second copy stream while step i+1 computes.  Events keep
    every buffer set's reuse ordered (4 rotating sets).  Returns the elapsed ms
    from the first upload to the last download, timed with events recorded on
    the compute stream after it joined both copy streams."""
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(sets)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_done, ev_out = {}, {}, {}
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up.wait_stream(comp)
    down.wait_stream(comp)
    start.record(up)

    def upload(i):
        s = sets[i % n]
        if i - n in ev_done:                 # the set's previous step has finished reading it
            up.wait_event(ev_done[i - n])
        with torch.cuda.stream(up):
            for name in ("x", "q_nope", "q_rope"):
                s[name].copy_(s[name + "_host"], non_blocking=True)
        ev_in[i] = ev(); ev_in[i].record(up)

    upload(0)
    for i in range(n_steps):
        if i + 1 < n_steps:
            upload(i + 1)
        comp.wait_event(ev_in[i])
        if i - n in ev_out:                  # the set's previous output has been downloaded
            comp.wait_event(ev_out[i - n])
        step(sets[i % n])
        ev_done[i] = ev(); ev_done[i].record(comp)
        down.wait_event(ev_done[i])
        with torch.cuda.stream(down):
            sets[i % n]["out_host"].copy_(sets[i % n]["out"], non_blocking=True)
        ev_out[i] = ev(); ev_out[i].record(down)
    comp.wait_stream(up)
    comp.wait_stream(down)
    stop.record(comp)
    torch.cuda.synchronize()
    return start.elapsed_time(stop)


def run_gpu(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from mla_latent_kv_write_b200 import build as vb
    from mla_latent_kv_write_b200 import videomla as V
    if rank == 0:
        vb.build()
    barrier(world)
    V.load_library()
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    Nk = wl.slots * T_f
    sets = make_sets(dev, N_SETS)
    fl_attn = flops_attention(d, wl.batch, wl.n_query, Nk)
    fl_cw = flops_cache_write(d, wl.batch, wl.n_query)
    fl_step = fl_attn + fl_cw

    for i in range(args.warmup):
        step(sets[i % N_SETS])
    barrier(world)
    if V.device_status(reset=True) != V.OK:
        raise RuntimeError("a kernel reported a timed-out device wait during warm-up")

    # ---- timed region: K steps, per-kernel events on the launch stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        start.record()
        for i in range(args.steps):
            step(sets[i % N_SETS], evs[i])
        stop.record()
        barrier(world)
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local, world)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    cw_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    clocks = clk.summary()

    s0 = sets[0]
    h2d_bytes = sum(s0[n].numel() * s0[n].element_size() for n in ("x", "q_nope", "q_rope"))
    d2h_bytes = s0["out"].numel() * s0["out"].element_size()

    # ---- end to end through host buffers (uploads / downloads pipelined with compute)
    run_e2e(sets, max(1, args.warmup))
    barrier(world)
    e2e_local = run_e2e(sets, args.steps)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_local, world)
    if V.device_status(reset=True) != V.OK:
        raise RuntimeError("a kernel reported a timed-out device wait")

    # ---- cache_write on a 30-layer stack (494 MB > L2), for its HBM roofline
    cw_stack = cache_write_stack(dev)
    cw_batched = cache_write_batched(dev) if world == 1 and not args.no_side else None
    del sets
    side = side_workloads(dev, measured_peaks()[0]["bf16_tflops"]) if world == 1 and not args.no_side else {}

    h2d = h2d_bytes
    d2h = d2h_bytes

    if rank == 0:
        peaks, peak_src = measured_peaks()
        sm = clocks.get("sm_mhz")
        sustained = sm is not None and sm < 1700.0
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        achieved = fl_attn / (attn_ms * 1e-3) / 1e12
        value = job_throughput(world, fl_step, ms, args.steps) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(world),
            "roofline": {"bound": "tensor", "kernel": "attention_kernel", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": f"{peak_src} bf16 {'sustained' if sustained else 'burst'} "
                                      f"(median SM clock {sm} MHz)",
                         "traffic": ncu_traffic("attention_kernel"),
                         "algorithmic_flops_per_launch": fl_attn},
            "attention_ms": attn_ms, "cache_write_ms": cw_ms,
            "query_tokens_per_s": job_throughput(world, wl.n_query, ms, args.steps),
            "explicit_mha_equivalent_tflops": flops_explicit_equivalent(d, wl.batch, wl.n_query, Nk)
            / (attn_ms * 1e-3) / 1e12,
            "cache_write_stack": cw_stack,
            "cache_write_batched": cw_batched,
            **side,
            "e2e": {"value": job_throughput(world, fl_step, e2e_ms, args.steps) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": e2e_ms / args.steps,
                    "pipelining": "step i+1 upload and step i-1 download overlap step i's kernels"},
            "clocks": clocks,
            "gpu_launches": 3 * args.steps,  # cache_write, window pre-pass, attention
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_sample()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _time_attention_calls(calls, reps: int):
    """Mean ms of one call of each of ``calls`` (closures launching one attention
    call), cycled ``reps`` times after a warm-up round; CUDA events on the
    current stream, which is the stream the calls launch on."""
    for c in calls:
        c()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        for c in calls:
            c()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / (reps * len(calls))


def side_workloads(dev, peak: float):
    """Attention on the pages' inference cache (one sink frame + a FIFO of six,
    App. D.4) and on every (d_c, d_rope) point of the rank / RoPE sweep (3 query
    frames vs a 21-frame window); each with 4 rotating input sets."""
    from mla_latent_kv_write_b200 import videomla as V
    wl = WORKLOAD
    res = {}

    def make(d, slots, n_sink, k):
        T_f = d.tokens_per_frame
        seed = I.seed_for(5, k, slots)
        w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
        q = {n: t.to(dev) for n, t in I.queries(d, 1, wl.n_query, seed + 1).items()}
        cache = I.latent_cache(d, 1, slots, seed + 2).to(dev)
        sink = I.latent_cache(d, 1, n_sink, seed + 3).to(dev) if n_sink else None
        ws = torch.empty(V.workspace_size(d, slots, 0, slots, 1, n_sink), dtype=torch.uint8, device=dev)
        out = torch.empty(1, wl.n_query, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev)
        return lambda: V.attention(q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, d, slots, 0, slots,
                                   out=out, workspace=ws, sink=sink)

    d = wl.dims
    calls = [make(d, 6, 1, k) for k in range(N_SETS)]
    ms = _time_attention_calls(calls, 10)
    Nk = 7 * d.tokens_per_frame
    tf = flops_attention(d, 1, wl.n_query, Nk) / (ms * 1e-3) / 1e12
    res["sink_window"] = {"workload": "Wan layer, 1 sink frame + FIFO of 6 frames (10920 keys), 4680 queries",
                          "ms": ms, "tflops": tf, "frac": tf / peak}
    del calls
    sweep = []
    for d_c, d_rope in I.SWEEP_POINTS:
        ds = I.sweep_dims(d_c, d_rope)
        calls = [make(ds, wl.slots, 0, k) for k in range(2)]
        ms = _time_attention_calls(calls, 5)
        tf = flops_attention(ds, 1, wl.n_query, wl.slots * ds.tokens_per_frame) / (ms * 1e-3) / 1e12
        sweep.append({"d_c": d_c, "d_rope": d_rope, "ms": ms, "tflops": tf, "frac": tf / peak})
        del calls
    res["sweep_attention"] = sweep
    torch.cuda.empty_cache()
    lat = next((x["ms"] for x in sweep if (x["d_c"], x["d_rope"]) == (d.d_c, d.d_rope)), None)
    res["dense_mha"] = dense_mha(dev, d, wl.n_query, wl.slots * d.tokens_per_frame, latent_ms=lat)
    res["layer_step"] = layer_step(dev, peak)
    res["projection_ab"] = projection_ab(dev)
    res["rolling"] = rolling_steps(dev, peak)
    res["long_window"] = long_window(dev, peak)
    return res


def rolling_steps(dev, peak: float):
    """The 40-step rolling workload: each step writes one frame (1560 tokens)
    into the 21-slot ring and attends its 1560 queries over the valid window;
    steps 20-39 (full, wrapping window) are timed back to back."""
    from mla_latent_kv_write_b200 import videomla as V
    wl = I.WORKLOADS["rolling"]
    d = wl.dims
    T_f = d.tokens_per_frame
    seed = I.seed_for(wl.index, 0, 0)
    w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
    xs = [I.tokens(d, wl.batch, T_f, seed + 100 + s).to(dev) for s in range(4)]
    qs = [{n: t.to(dev) for n, t in I.queries(d, wl.batch, T_f, seed + 200 + s).items()} for s in range(4)]
    cache = torch.zeros(wl.batch, wl.slots * T_f, d.cache_width, dtype=torch.bfloat16, device=dev)
    out = torch.empty(wl.batch, T_f, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev)

    def do_step(s):
        slot = s % wl.slots
        n_valid = min(s + 1, wl.slots)
        oldest = 0 if s + 1 <= wl.slots else (slot + 1) % wl.slots
        V.cache_write(xs[s % 4], w["W_dkv"], w["W_kr"], w["gamma"], cache, d, wl.slots, slot)
        q = qs[s % 4]
        V.attention(q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, d, wl.slots, oldest, n_valid, out=out)

    def run(mode):
        with V.attention_tiling(mode):
            cache.zero_()
            for s in range(20):
                do_step(s)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for s in range(20, wl.steps):
                do_step(s)
            b.record()
            torch.cuda.synchronize()
        return a.elapsed_time(b) / (wl.steps - 20)

    ms_head = run(V.TILING_PER_HEAD)  # A/B: one CTA per (query tile, head), split-KV over 3 CTAs
    ms = run(V.TILING_AUTO)           # the library's choice: head-packed tiles
    fl = flops_cache_write(d, wl.batch, T_f) + flops_attention(d, wl.batch, T_f, wl.slots * T_f)
    ctas = (d.n_heads * T_f + 127) // 128 * wl.batch
    return {"workload": "rolling: 1 frame (1560 tokens) per step into a 21-slot ring, steps 20-39 timed",
            "ms_per_step": ms, "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / peak,
            "attention_ctas": ctas, "tiling": "head-packed (128 consecutive (head, query) rows per CTA)",
            "per_head_tiles": {"ms_per_step": ms_head, "frac": fl / (ms_head * 1e-3) / 1e12 / peak,
                               "attention_ctas": "156 units x 3-way split-KV"}}


def long_window(dev, peak: float):
    """Minute-scale window: batch 2, 63-frame ring (98,280 keys), 4680 queries."""
    from mla_latent_kv_write_b200 import videomla as V
    wl = I.WORKLOADS["long"]
    d = wl.dims
    T_f = d.tokens_per_frame
    calls = []
    for k in range(2):
        seed = I.seed_for(wl.index, k, 0)
        w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
        q = {n: t.to(dev) for n, t in I.queries(d, wl.batch, wl.chunk * T_f, seed + 1).items()}
        cache = I.latent_cache(d, wl.batch, wl.slots, seed + 2).to(dev)
        out = torch.empty(wl.batch, wl.chunk * T_f, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev)
        calls.append(lambda w=w, q=q, cache=cache, out=out: V.attention(
            q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, d, wl.slots, 0, wl.slots, out=out))
    ms = _time_attention_calls(calls, 3)
    fl = flops_attention(d, wl.batch, wl.chunk * T_f, wl.slots * T_f)
    return {"workload": "long: batch 2, 63-frame ring (98280 keys), 4680 queries", "ms": ms,
            "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / peak}


def layer_step(dev, peak: float):
    """One whole attention-layer step on the Wan chunk: query path (Eq. 3-4, 6),
    cache write, latent attention over the 21-frame window, output projection;
    2 rotating input sets, CUDA events around the four calls."""
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    M = wl.n_query
    import ctypes
    lib = V.load_library()
    cd = V.c_dims(d)
    q_ws = int(lib.videomla_query_projection_workspace_size(ctypes.byref(cd), d.d_q, 1, M))
    a_ws = V.workspace_size(d, wl.slots, 0, wl.slots, 1, n_query=M)
    side = torch.cuda.Stream(device=dev)
    calls, calls_ovl = [], []
    for k in range(2):
        seed = I.seed_for(6, k, 0)
        w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
        pw = {n: t.to(dev) for n, t in I.projection_weights(d, seed + 1).items()}
        x = I.tokens(d, 1, M, seed + 2).to(dev)
        cache = I.latent_cache(d, 1, wl.slots, seed + 3).to(dev)
        qn = torch.empty(1, M, d.n_heads, d.d_nope, dtype=torch.bfloat16, device=dev)
        qr = torch.empty(1, M, d.n_heads, d.d_rope, dtype=torch.bfloat16, device=dev)
        o = torch.empty(1, M, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev)
        y = torch.empty(1, M, d.d_model, dtype=torch.bfloat16, device=dev)
        qw = torch.empty(max(q_ws, 16), dtype=torch.uint8, device=dev)
        aw = torch.empty(max(a_ws, 16), dtype=torch.uint8, device=dev)

        def call(w=w, pw=pw, x=x, cache=cache, qn=qn, qr=qr, o=o, y=y, qw=qw, aw=aw):
            V.query_projection(x, pw["W_dq"], pw["gamma_q"], pw["W_uq"], pw["W_qr"], d, q_nope=qn, q_rope=qr,
                               workspace=qw)
            V.cache_write(x, w["W_dkv"], w["W_kr"], w["gamma"], cache, d, wl.slots, wl.prefill)
            V.attention(qn, qr, w["W_uk"], w["W_uv"], cache, d, wl.slots, 0, wl.slots, out=o, workspace=aw)
            V.output_projection(o, pw["W_O"], d, y=y)

        def call_ovl(w=w, pw=pw, x=x, cache=cache, qn=qn, qr=qr, o=o, y=y, qw=qw, aw=aw):
            # the query path and the cache write both only read x: the query path on a
            # second stream, the attention waits for both
            main = torch.cuda.current_stream(dev)
            side.wait_stream(main)
            V.query_projection(x, pw["W_dq"], pw["gamma_q"], pw["W_uq"], pw["W_qr"], d, q_nope=qn, q_rope=qr,
                               workspace=qw, stream=side)
            V.cache_write(x, w["W_dkv"], w["W_kr"], w["gamma"], cache, d, wl.slots, wl.prefill)
            main.wait_stream(side)
            V.attention(qn, qr, w["W_uk"], w["W_uv"], cache, d, wl.slots, 0, wl.slots, out=o, workspace=aw)
            V.output_projection(o, pw["W_O"], d, y=y)
        calls.append(call)
        calls_ovl.append(call_ovl)
    ms = _time_attention_calls(calls, 10)
    ms_ovl = _time_attention_calls(calls_ovl, 10)
    fl_q = 2.0 * M * (d.d_model * d.d_q + d.d_q * d.n_heads * (d.d_nope + d.d_rope))
    fl_o = 2.0 * M * d.n_heads * d.d_v * d.d_model
    fl = fl_q + flops_cache_write(d, 1, M) + flops_attention(d, 1, M, wl.slots * T_f) + fl_o
    return {"workload": "Wan layer step: query path + cache write of 3 frames + attention over 21 frames "
                        "+ output projection, 4680 tokens", "ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
            "frac": fl / (ms * 1e-3) / 1e12 / peak, "flops": fl, "projection_flops": fl_q + fl_o,
            "overlapped": {"how": "query path on a second stream beside the cache write, joined before "
                                  "the attention", "ms": ms_ovl, "tflops": fl / (ms_ovl * 1e-3) / 1e12,
                           "frac": fl / (ms_ovl * 1e-3) / 1e12 / peak}}


def projection_ab(dev):
    """The two re-associations the pages give for inference, each timed against
    the order this library uses (Wan chunk, 4680 tokens, 12 heads, d_c 192):
      output side (App. E Eq. 10-11): y = sum_h B_h o_lat,h with B_h = W_O,h W_uv,h
        [d_model x d_c] -- one GEMM with K = H d_c = 2304 on the per-head O_lat / l
        -- against the attention's W_uv epilogue + y = W_O [o_1 .. o_H] (K = H d_v
        = 1536);
      query side (Eq. 9): q_abs,h = A_h^T c^Q with A_h = W_uq,h^T W_uk,h
        [d_q x d_c] -- the up-projection GEMM widens from H d_nope = 1152 to
        H d_c = 2304 columns -- against q^nope = W_uq c^Q + the attention's
        in-kernel absorption.
    Each GEMM runs through the public entry points (the output projection with
    d_v := d_c, the query path with d_nope := d_c) on random weights of those
    shapes, 10 calls per CUDA graph.  The attention-side terms (W_uv epilogue,
    absorption) are counted in flops: each is under 0.2 % of the attention."""
    import dataclasses
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    M = wl.n_query
    g = torch.Generator().manual_seed(7100)

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(dev)
    out = {}
    # output side
    o = rnd(1, M, d.n_heads, d.d_v)
    W_O = rnd(d.d_model, d.n_heads * d.d_v, std=(d.n_heads * d.d_v) ** -0.5)
    y = torch.empty(1, M, d.d_model, dtype=torch.bfloat16, device=dev)
    d_b = dataclasses.replace(d, d_v=d.d_c)
    o_lat = rnd(1, M, d.n_heads, d.d_c)
    B = rnd(d.d_model, d.n_heads * d.d_c, std=(d.n_heads * d.d_c) ** -0.5)
    t_wo = _graph_time_ms(lambda: [V.output_projection(o, W_O, d, y=y) for _ in range(10)], 5) / 10
    t_b = _graph_time_ms(lambda: [V.output_projection(o_lat, B, d_b, y=y) for _ in range(10)], 5) / 10
    fl_wo = 2.0 * M * d.n_heads * d.d_v * d.d_model
    fl_uv = 2.0 * M * d.n_heads * d.d_c * d.d_v
    fl_b = 2.0 * M * d.n_heads * d.d_c * d.d_model
    out["output_side"] = {"built_W_O_gemm_ms": t_wo, "built_gflop": (fl_wo + fl_uv) / 1e9,
                          "B_h_gemm_ms": t_b, "B_h_gflop": fl_b / 1e9, "faster": "built" if t_wo <= t_b else "B_h"}
    # query side
    pw = {n: t.to(dev) for n, t in I.projection_weights(d, 7101).items()}
    x = rnd(1, M, d.d_model)
    d_a = dataclasses.replace(d, d_nope=d.d_c)
    A_t = rnd(d.n_heads * d.d_c, d.d_q, std=d.d_q ** -0.5)
    qn = torch.empty(1, M, d.n_heads, d.d_nope, dtype=torch.bfloat16, device=dev)
    qa = torch.empty(1, M, d.n_heads, d.d_c, dtype=torch.bfloat16, device=dev)
    qr = torch.empty(1, M, d.n_heads, d.d_rope, dtype=torch.bfloat16, device=dev)
    t_q = _graph_time_ms(lambda: [V.query_projection(x, pw["W_dq"], pw["gamma_q"], pw["W_uq"], pw["W_qr"], d,
                                                     q_nope=qn, q_rope=qr) for _ in range(10)], 5) / 10
    t_a = _graph_time_ms(lambda: [V.query_projection(x, pw["W_dq"], pw["gamma_q"], A_t, pw["W_qr"], d_a,
                                                     q_nope=qa, q_rope=qr) for _ in range(10)], 5) / 10
    fl_dq = 2.0 * M * d.d_model * d.d_q
    fl_q = fl_dq + 2.0 * M * d.d_q * d.n_heads * (d.d_nope + d.d_rope)
    fl_abs = 2.0 * M * d.n_heads * d.d_nope * d.d_c
    fl_a = fl_dq + 2.0 * M * d.d_q * d.n_heads * (d.d_c + d.d_rope)
    out["query_side"] = {"built_query_path_ms": t_q, "built_gflop": (fl_q + fl_abs) / 1e9,
                         "A_h_query_path_ms": t_a, "A_h_gflop": fl_a / 1e9, "faster": "built" if t_q <= t_a else "A_h"}
    return out


def dense_mha(dev, d, Nq: int, Nk: int, latent_ms: float):
    """The pages' dense baseline on the same shape ([VideoMLA] App. C.1): per-head
    K and V of 128 channels for every key, the 2 n_h d_h = 3072-scalar cache, through
    this library's dense kernel (``videomla_dense_attention``, parity-tested against
    the oracle's explicit form), and through torch's scaled-dot-product attention
    (cuDNN / flash) for reference.  Random K / V of that shape (2 sets of 2 x
    201 MB, larger than L2); flops 4 d_h per (q, k, h).  The latent call's time is
    passed in for the ratio."""
    import torch.nn.functional as F
    from mla_latent_kv_write_b200 import videomla as V
    dh = d.d_nope + d.d_rope
    g = torch.Generator(device="cpu").manual_seed(77)
    sets = []
    for _ in range(2):
        qn = torch.randn(1, Nq, d.n_heads, d.d_nope, generator=g).to(torch.bfloat16).to(dev)
        qr = torch.randn(1, Nq, d.n_heads, d.d_rope, generator=g).to(torch.bfloat16).to(dev)
        k = torch.randn(1, Nk, d.n_heads, dh, generator=g).to(torch.bfloat16).to(dev)
        v = torch.randn(1, Nk, d.n_heads, dh, generator=g).to(torch.bfloat16).to(dev)
        o = torch.empty(1, Nq, d.n_heads, dh, dtype=torch.bfloat16, device=dev)
        sets.append((qn, qr, k, v, o))
    calls = [lambda qn=qn, qr=qr, k=k, v=v, o=o: V.dense_attention(qn, qr, k, v, d, out=o)
             for qn, qr, k, v, o in sets]
    ms_ours = _time_attention_calls(calls, 5)
    backend = "default"
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        ctx = sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION])
        backend = "cudnn / flash / efficient (first available)"
    except Exception:  # older torch: its own choice
        import contextlib
        ctx = contextlib.nullcontext()
    lib_sets = [(torch.cat([qn, qr], -1).transpose(1, 2).contiguous(), k.transpose(1, 2).contiguous(),
                 v.transpose(1, 2).contiguous()) for qn, qr, k, v, _ in sets]
    with ctx:
        calls = [lambda q=q, k=k, v=v: F.scaled_dot_product_attention(q, k, v) for q, k, v in lib_sets]
        ms_lib = _time_attention_calls(calls, 5)
    fl = 4.0 * dh * Nq * Nk * d.n_heads
    del sets, lib_sets
    torch.cuda.empty_cache()
    return {"what": "dense multi-head attention on per-head K / V, same queries and window",
            "ours_ms": ms_ours, "ours_tflops": fl / (ms_ours * 1e-3) / 1e12,
            "library_backend": backend, "library_ms": ms_lib, "library_tflops": fl / (ms_lib * 1e-3) / 1e12,
            "latent_attention_ms": latent_ms,
            "latent_over_dense_time": None if latent_ms is None else latent_ms / ms_ours,
            "cache_bytes_per_token_layer": 2 * 2 * d.n_heads * dh,
            "latent_cache_bytes_per_token_layer": 2 * (d.d_c + d.d_rope),
            "dense_window_bytes": 2 * 2 * d.n_heads * dh * Nk, "latent_window_bytes": 2 * (d.d_c + d.d_rope) * Nk}


def _graph_time_ms(run, reps: int) -> float:
    """Best-of-``reps`` CUDA-event time of one replay of the calls ``run`` makes,
    captured into a CUDA graph so that the events time the GPU, not the Python
    launch loop (a 4680-token cache write takes microseconds, less than the host
    needs to prepare a call)."""
    run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            run()
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    evs = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    del graph
    return min(a.elapsed_time(b) for a, b in evs)


def cache_write_stack(dev, layers: int = 30, reps: int = 3):
    """cache_write over 30 independent layers (3-frame chunks, 494 MB of x +
    cache traffic > L2), timed back to back; HBM roofline of that kernel."""
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    n_tok = wl.chunk * T_f
    xs, caches, ws = [], [], []
    for l in range(layers):
        seed = I.seed_for(4, l, 0)
        xs.append(I.tokens(d, 1, n_tok, seed).to(dev))
        ws.append({k: v.to(dev) for k, v in I.layer_weights(d, seed).items()})
        caches.append(torch.zeros(1, wl.slots * T_f, d.cache_width, dtype=torch.bfloat16, device=dev))

    def run():
        for l in range(layers):
            V.cache_write(xs[l], ws[l]["W_dkv"], ws[l]["W_kr"], ws[l]["gamma"], caches[l], d, wl.slots, wl.prefill)
    ms = _graph_time_ms(run, reps) / layers
    by = bytes_cache_write(d, 1, n_tok)
    gbs = by / (ms * 1e-3) / 1e9
    peaks, src = measured_peaks()
    return {"layers": layers, "timing": "30 calls replayed from one CUDA graph, best of 3",
            "ms_per_layer": ms, "bytes_per_layer": by, "achieved_gbs": gbs,
            "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"{src} HBM copy",
            "tflops": flops_cache_write(d, 1, n_tok) / (ms * 1e-3) / 1e12,
            "roofline": {"bound": "hbm", "kernel": "cache_write_cluster_kernel", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "peak_kind": f"{src} HBM copy", "algorithmic_bytes_per_launch": by,
                         "traffic": ncu_traffic("cache_write_cluster_kernel")}}


def cache_write_batched(dev, batches=(1, 2, 4, 8), reps: int = 5):
    """The cache write of a 3-frame chunk for batch 1, 2, 4 and 8 requests in one
    call: three rotating input sets (x and ring differ per call, > L2 at batch
    >= 4), six calls per CUDA graph.  With more 128-token tiles than half the SMs
    the call runs the persistent stream kernel."""
    from mla_latent_kv_write_b200 import videomla as V
    wl, d = WORKLOAD, WORKLOAD.dims
    T_f = d.tokens_per_frame
    n_tok = wl.chunk * T_f
    peaks, src = measured_peaks()
    out = []
    for B in batches:
        xs = [I.tokens(d, B, n_tok, I.seed_for(4, 0, 50 + k)).to(dev) for k in range(3)]
        w = {k: v.to(dev) for k, v in I.layer_weights(d, I.seed_for(4, 0, 60)).items()}
        caches = [torch.zeros(B, wl.slots * T_f, d.cache_width, dtype=torch.bfloat16, device=dev) for _ in range(3)]

        def run():
            for k in range(6):
                V.cache_write(xs[k % 3], w["W_dkv"], w["W_kr"], w["gamma"], caches[k % 3], d, wl.slots,
                              wl.prefill)
        ms = _graph_time_ms(run, reps) / 6
        by = bytes_cache_write(d, B, n_tok)
        tiles = B * ((n_tok + 127) // 128)
        out.append({"batch": B, "tiles": tiles,
                    "kernel": "cache_write_cluster_kernel" if 2 * tiles <= 148 else "cache_write_stream_kernel",
                    "us_per_call": ms * 1e3, "achieved_gbs": by / (ms * 1e-3) / 1e9,
                    "frac": by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
        del xs, caches
    return out


def profile_sweep(spec: str) -> int:
    """Three attention calls on one (d_c, d_rope) point of the rank / RoPE sweep
    (3 query frames vs a 21-frame window, the bench's seeded inputs), nothing
    timed: a short command for a profiler to capture one launch of that kernel."""
    from mla_latent_kv_write_b200 import videomla as V
    d_c, d_rope = (int(v) for v in spec.split(","))
    if (d_c, d_rope) not in I.SWEEP_POINTS:
        raise SystemExit(f"--profile-sweep: {spec} is not one of {I.SWEEP_POINTS}")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    V.load_library()
    wl = WORKLOAD
    d = I.sweep_dims(d_c, d_rope)
    seed = I.seed_for(5, 0, wl.slots)
    w = {n: t.to(dev) for n, t in I.layer_weights(d, seed).items()}
    q = {n: t.to(dev) for n, t in I.queries(d, 1, wl.n_query, seed + 1).items()}
    cache = I.latent_cache(d, 1, wl.slots, seed + 2).to(dev)
    ws = torch.empty(V.workspace_size(d, wl.slots, 0, wl.slots, 1), dtype=torch.uint8, device=dev)
    out = torch.empty(1, wl.n_query, d.n_heads, d.d_v, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        V.attention(q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, d, wl.slots, 0, wl.slots,
                    out=out, workspace=ws)
    torch.cuda.synchronize()
    if V.device_status(reset=True) != V.OK:
        raise RuntimeError("a kernel reported a timed-out device wait")
    print(f"profile-sweep {d_c},{d_rope}: 3 attention calls done")
    return 0


def profile_dense() -> int:
    """Three calls of the dense multi-head attention baseline at the Wan layer
    shape (random per-head K / V of the 21-frame window), nothing timed: a short
    command for a profiler to capture one launch of that kernel."""
    from mla_latent_kv_write_b200 import videomla as V
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    V.load_library()
    wl, d = WORKLOAD, WORKLOAD.dims
    Nk = wl.slots * d.tokens_per_frame
    g = torch.Generator().manual_seed(78)
    qn = torch.randn(1, wl.n_query, d.n_heads, d.d_nope, generator=g).to(torch.bfloat16).to(dev)
    qr = torch.randn(1, wl.n_query, d.n_heads, d.d_rope, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(1, Nk, d.n_heads, 128, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(1, Nk, d.n_heads, 128, generator=g).to(torch.bfloat16).to(dev)
    for _ in range(3):
        V.dense_attention(qn, qr, k, v, d)
    torch.cuda.synchronize()
    if V.device_status(reset=True) != V.OK:
        raise RuntimeError("a kernel reported a timed-out device wait")
    print("profile-dense: 3 dense attention calls done")
    return 0


def profile_projection() -> int:
    """Three calls of the output projection (W_O over the 12 heads' outputs) at
    the Wan chunk shape (4680 tokens), nothing timed: a short command for a
    profiler to capture one launch of the pair GEMM."""
    from mla_latent_kv_write_b200 import videomla as V
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    V.load_library()
    d, M = WORKLOAD.dims, WORKLOAD.n_query
    pw = {n: t.to(dev) for n, t in I.projection_weights(d, 77).items()}
    g = torch.Generator().manual_seed(79)
    o = torch.randn(1, M, d.n_heads, d.d_v, generator=g).to(torch.bfloat16).to(dev)
    y = torch.empty(1, M, d.d_model, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        V.output_projection(o, pw["W_O"], d, y=y)
    torch.cuda.synchronize()
    if V.device_status(reset=True) != V.OK:
        raise RuntimeError("a kernel reported a timed-out device wait")
    print("profile-projection: 3 output projection calls done")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the sink-window and sweep side measurements")
    ap.add_argument("--profile-projection", action="store_true",
                    help="only run three output-projection calls at the Wan shape (for a profiler), then exit")
    ap.add_argument("--profile-dense", action="store_true",
                    help="only run three dense-baseline attention calls (for a profiler), then exit")
    ap.add_argument("--profile-sweep", metavar="D_C,D_ROPE",
                    help="only run three attention calls of one rank-sweep point (for a profiler), then exit")
    args = ap.parse_args()
    if args.profile_sweep:
        return profile_sweep(args.profile_sweep)
    if args.profile_dense:
        return profile_dense()
    if args.profile_projection:
        return profile_projection()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
