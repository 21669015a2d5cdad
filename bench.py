#!/usr/bin/env python
"""Benchmark of the sparse MXFP4 MoE decode layer (libmoe_decode.so) on B200.

One step = one moe_layer_forward of the workload (router GEMV + top-k +
bucketing, routed MXFP4 SwiGLU experts, the shared expert, down projection
fused with the combine and residual add) on one batch of
seeded synthetic tokens; a pool of distinct tokens makes every step route to
a different expert set.  Weights and inputs are resident in HBM before the
timed region; L2 is flushed (256 MiB write) between steps, outside the
per-step CUDA events.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1|2|3|4] [--impl ours|reference]

--gpus N > 1 runs under torchrun as N independent replicas (the layer does
not shard); value = the bytes all ranks moved / the slowest rank's time.
--impl reference times the CPU oracle on the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE decode layer achieved HBM GB/s (counted bytes per layer-step / device time per layer-step)"
UNIT = "GB/s"
WORKLOAD_DEFAULT = 1
POOL = 64  # distinct token batches cycled through the steps (--pool)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=WORKLOAD_DEFAULT)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flags", type=int, default=0, help="MOE_FLAG_* bits for ablations")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling aid: fewer routed experts (same per-step work, smaller footprint)")
    ap.add_argument("--pool", type=int, default=64, help="distinct token batches cycled through the steps")
    return ap.parse_args()


def workload_desc(cfg):
    return (f"{cfg.name}: one MoE decode layer, hidden {cfg.hidden}, {cfg.n_experts} routed experts top-{cfg.top_k}, "
            f"expert intermediate {cfg.inter} (MXFP4 E2M1 + E8M0/32), shared expert intermediate "
            f"{cfg.shared_inter} (bf16), batch {cfg.batch}" + (f", Zipf({cfg.zipf_s}) router bias" if cfg.zipf_s else ""))


# ---------------------------------------------------------------- clocks ----
def _load_nvml():
    import pynvml
    return pynvml


class ClockSampler:
    """SM clock and clock-event (throttle) reasons while the timed regions run.

    NVML, read in-process by a thread every 5 ms (reading only: no setting is
    changed); only samples taken between begin() and end() count.  If NVML
    cannot be used, nvidia-smi's 50 ms loop instead, started before the
    warm-up and waited for, so that it is already sampling when timing
    starts."""
    PERIOD_S = 0.005
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                   ("sw_power_cap", 0x4))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, uuid=None):
        self.gpu = gpu_index
        self.uuid = uuid
        self.nv = None
        self.proc = None
        self.lines = []
        self.samples = []       # (perf_counter, sm MHz, reason bits)
        self.windows = []       # (begin, end) of the timed regions
        self._open = None
        self._halt = threading.Event()

    # -- NVML --------------------------------------------------------------
    def _nvml_start(self):
        nv = _load_nvml()
        nv.nvmlInit()
        try:
            h = None
            if self.uuid:
                u = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
                try:
                    h = nv.nvmlDeviceGetHandleByUUID(u)
                except Exception:
                    h = None
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            try:
                nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons
            except Exception:
                reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._read = lambda: (time.perf_counter(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                  int(reasons(h)))
            self.samples.append(self._read())     # a failing read fails here, not in the thread
        except Exception:
            try:
                nv.nvmlShutdown()
            except Exception:
                pass
            raise
        self.nv = nv
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        while not self._halt.wait(self.PERIOD_S):
            try:
                self.samples.append(self._read())
            except Exception:
                return

    # -- nvidia-smi ----------------------------------------------------------
    def _smi_start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._smi_read, daemon=True)
        self.thread.start()
        t0 = time.perf_counter()
        while not self.lines and self.proc.poll() is None and time.perf_counter() - t0 < 3.0:
            time.sleep(0.01)

    def _smi_read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _smi_stop(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = [n for n, _ in self.REASON_BITS]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 50 ms, whole run"}

    # -- public ----------------------------------------------------------------
    def start(self):
        try:
            self._nvml_start()
        except Exception:
            self.nv = None
            self._smi_start()

    def begin(self):
        self._open = time.perf_counter()

    def end(self):
        if self._open is not None:
            self.windows.append((self._open, time.perf_counter()))
            self._open = None

    def stop(self):
        if self.nv is not None:
            self._halt.set()
            self.thread.join(timeout=2.0)
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass
            inside = [s for s in self.samples if any(a <= s[0] <= b for a, b in self.windows)]
            bits = 0
            for s in inside:
                bits |= s[2]
            return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
                    "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(n for n, b in self.REASON_BITS if bits & b),
                    "samples": len(inside), "source": "NVML, 5 ms, timed regions only"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source (NVML and nvidia-smi unavailable)"],
                    "samples": 0}
        return self._smi_stop()


# ------------------------------------------------------------- helpers ------
def _code_only(src):
    """C++ source with comments and blank lines removed (string literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(l.rstrip() for l in "".join(out).splitlines() if l.strip())


def kernel_source_sha():
    """Hash of the code (comments ignored) of the sources that build the
    routed gate/up kernel: a recorded ncu traffic figure stays valid as long
    as this hash is unchanged."""
    h = hashlib.sha256()
    for f in ("kernels.cuh", "gemv.cuh", "ptx.cuh", "moe_decode.cu"):
        with open(os.path.join(ROOT, "sparse_moe_decode_router_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_tag, workload):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, if it was taken on the current kernel sources."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    sha = kernel_source_sha()
    for fn in sorted(os.listdir(d)):
        if not fn.endswith(".md"):
            continue
        txt = open(os.path.join(d, fn)).read()
        m = re.search(r"traffic_record:\s*kernel=(\S+)\s+workload=(\S+)\s+sha=(\w+)\s+bytes_per_launch=(\d+)", txt)
        if m and m.group(1) == kernel_tag and m.group(2) == workload and m.group(3) == sha:
            return int(m.group(4))
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def max_over_ranks(values, device="cpu"):
    """Element-wise maximum of `values` over all ranks (the slowest replica
    sets the job's time); identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_value(world, total_bytes_per_rank, slowest_ms):
    """Whole-job GB/s of N replicas: the bytes all ranks moved / the slowest rank's time."""
    return world * total_bytes_per_rank / (slowest_ms * 1e-3) / 1e9


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world} (launch N>1 with torchrun)")
    return world, rank, local


# -------------------------------------------------------- reference arm -----
def run_reference(args, cfg):
    """The oracle (fp64 CPU) on the same workload, rank 0 only."""
    world, rank, local = dist_setup(args.gpus)
    if rank != 0:
        return
    import torch
    import oracle
    from synth.workload import make_device_layer, residual_tokens
    torch.cuda.set_device(local)
    dl = make_device_layer(cfg, 0)
    B = cfg.batch
    threads = os.cpu_count() or 1
    shared = dl.host_shared()
    times, counted = [], []
    total = min(args.warmup, 1) + args.steps
    t_start = time.perf_counter()
    for i in range(total):
        if times and time.perf_counter() - t_start > 90.0:
            break              # bounded sample: the oracle needs ~1 s per full layer-step
        ids = [((i % POOL) * B) + b for b in range(B)]
        x_h, _ = dl.tokens(ids)
        r_h, _ = residual_tokens(cfg, ids)
        rt = oracle.routing(x_h, dl.router_w_host, dl.bias_host, cfg.top_k)
        sel = np.unique(rt["topk_idx"])
        gc, gs, dc, ds = dl.host_experts(sel)
        t0 = time.perf_counter()
        oracle.layer(x_h, r_h, dl.router_w_host, dl.bias_host, gc, gs, dc, ds, shared[0], shared[1],
                     cfg.top_k, experts=sel, n_threads=threads)
        dt = time.perf_counter() - t0
        if i >= min(args.warmup, 1):
            times.append(dt)
            counted.append(cfg.counted_bytes(len(sel)))
    sec = statistics.mean(times)
    value = statistics.mean(counted) / sec / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "parallelism": "rank 0 only (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{len(times)} of {args.steps} steps timed (90 s cap), each a full "
                                       f"layer-step of batch {B} (fp64 C++ oracle, OpenMP over {threads} threads)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- our arm ----
class _DevPtr:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3}


def run_ours(args, cfg):
    world, rank, local = dist_setup(args.gpus)
    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from sparse_moe_decode_router_b200 import api
    from synth.workload import make_device_layer, residual_tokens

    api.load_library()
    B, H, k = cfg.batch, cfg.hidden, cfg.top_k
    dl = make_device_layer(cfg, 0)
    c = api.moe_layer_config(cfg.hidden, cfg.n_experts, cfg.top_k, cfg.inter, cfg.shared_inter, B, args.flags)
    handle = api.moe_layer_create(c, dl.weights_struct())
    pool_x, pool_r, pool_xh, pool_rh = [], [], [], []
    for p in range(POOL):
        ids = [p * B + b for b in range(B)]
        xh, xd = dl.tokens(ids)
        rh, rd = residual_tokens(cfg, ids)
        pool_x.append(xd)
        pool_r.append(rd)
        pool_xh.append(torch.from_numpy(xh.view(np.int16)).pin_memory())
        pool_rh.append(torch.from_numpy(rh.view(np.int16)).pin_memory())
    out = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
    out_h = torch.empty((B, H), dtype=torch.int16).pin_memory()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    plan = api.moe_layer_routing(handle)
    n_act_view = torch.as_tensor(_DevPtr(plan.n_active, (1,), "<i4"), device="cuda")

    # experts touched by each pool batch (read back before any timing)
    n_active = []
    for p in range(POOL):
        api.moe_layer_forward(handle, None, pool_x[p], pool_r[p], out, B, stream)
        n_active.append(int(n_act_view.cpu()[0]))
    torch.cuda.synchronize()
    if api.moe_layer_last_device_error(handle) != api.MOE_OK:
        raise SystemExit("device-side error during warm-up")

    def step_bytes(i):
        return cfg.counted_bytes(n_active[i % POOL])

    # routed gate/up kernel: codes + scales of the active experts, x in, h out (fp32)
    def gate_up_bytes(i):
        na = n_active[i % POOL]
        return na * 2 * cfg.inter * (H // 2 + H // 32) + B * H * 2 + B * k * cfg.inter * 4

    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(local, uuid)
    sampler.start()
    for i in range(args.warmup):
        flush.zero_()
        api.moe_layer_forward(handle, None, pool_x[i % POOL], pool_r[i % POOL], out, B, stream)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    pr = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in pr:  # materialise the CUDA events before handing them to the library
        a.record(stream)
        b.record(stream)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.begin()
    for i in range(K):
        flush.zero_()
        api.moe_layer_set_probe(handle, pr[i][0], pr[i][1])
        ev[i][0].record(stream)
        api.moe_layer_forward(handle, None, pool_x[i % POOL], pool_r[i % POOL], out, B, stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    sampler.end()
    if dist is not None:
        dist.barrier()
    api.moe_layer_set_probe(handle, None, None)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    gu_ms = [a.elapsed_time(b) for a, b in pr]

    # end to end through the host-buffer entry point (pinned host memory)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    sampler.begin()
    for i in range(K):
        flush.zero_()
        e2e_ev[i][0].record(stream)
        api.moe_layer_forward_host(handle, pool_xh[i % POOL], pool_rh[i % POOL], out_h, B, stream)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    sampler.end()
    clocks = sampler.stop()
    e2e_ms = [a.elapsed_time(b) for a, b in e2e_ev]
    if api.moe_layer_last_device_error(handle) != api.MOE_OK:
        raise SystemExit("device-side error during the timed region")

    total_ms = sum(step_ms)
    total_bytes = sum(step_bytes(i) for i in range(K))
    e2e_total = sum(e2e_ms)
    gu_avg_s = statistics.mean(gu_ms) * 1e-3
    gu_bytes = statistics.mean([gate_up_bytes(i) for i in range(K)])
    if dist is not None:
        total_ms, e2e_total = max_over_ranks([total_ms, e2e_total], "cuda")
    api.moe_layer_destroy(handle)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_per_step = total_ms / K
    value = job_value(world, total_bytes, total_ms)
    peak, peak_src = measured_peaks()
    achieved = gu_bytes / gu_avg_s / 1e9
    traffic = recorded_traffic("routed_gate_up", cfg.name)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded Philox4x32-10 draws; random-init weights of the full-size layer)",
        "config": {"workload": workload_desc(cfg), "batch": B, "parallelism": f"replicas x{world}",
                   "l2": "flushed between steps (256 MiB write, outside the per-step CUDA events)",
                   "token_pool": POOL, "flags": args.flags},
        "us_per_step": round(ms_per_step * 1e3, 2),
        "tokens_per_s": round(world * B * K / (total_ms * 1e-3), 1),
        "counted_bytes_per_step": int(total_bytes / K),
        "n_active_mean": statistics.mean(n_active[i % POOL] for i in range(K)),
        "frac_of_measured_hbm": round(value / world / peak, 4),
        "roofline": {"kernel": "routed_gate_up", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": int(gu_bytes),
                     "avg_launch_us": round(gu_avg_s * 1e6, 2)},
        "e2e": {"value": round(world * total_bytes / (e2e_total * 1e-3) / 1e9, 2), "unit": UNIT,
                "h2d_bytes_per_step": 2 * B * H * 2, "d2h_bytes_per_step": B * H * 2,
                "us_per_step": round(e2e_total / K * 1e3, 2)},
        "gpu_launches": launches_per_step(cfg, args.flags) * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, dl)
    print(json.dumps(line), flush=True)


def launches_per_step(cfg, flags):
    """Kernels of this library one moe_layer_forward launches: router GEMV and
    top-k; the shared expert's gate/up and down; then, for batches of one to
    eight (or with the grouped path off), routed gate/up and down+combine;
    above eight, the grouped tensor-core path: an activation-staging kernel
    and a grouped MMA kernel per projection, then the combine.  The grouped
    path is taken when both reduction lengths are multiples of 256 (the
    full-size and test shapes)."""
    from sparse_moe_decode_router_b200.api import MOE_FLAG_NO_GROUPED
    n = 2 + (2 if cfg.shared_inter > 0 else 0)
    grouped = (cfg.batch > 8 and not (flags & MOE_FLAG_NO_GROUPED) and cfg.hidden % 256 == 0
               and cfg.inter % 256 == 0)
    return n + (5 if grouped else 2)


def cpu_baseline(cfg, dl):
    """The oracle as it stands on the host cores, on a bounded sample of the
    same workload: whole layer-steps until ~10 s of CPU work (at least one)."""
    import oracle
    from synth.workload import residual_tokens
    threads = os.cpu_count() or 1
    B = cfg.batch
    shared = dl.host_shared()
    spent, n, nbytes = 0.0, 0, 0
    while n < 1 or (spent < 10.0 and n < 64):
        ids = [((n % POOL) * B) + b for b in range(B)]
        x_h, _ = dl.tokens(ids)
        r_h, _ = residual_tokens(cfg, ids)
        rt = oracle.routing(x_h, dl.router_w_host, dl.bias_host, cfg.top_k)
        sel = np.unique(rt["topk_idx"])
        gc, gs, dc, ds = dl.host_experts(sel)
        t0 = time.perf_counter()
        oracle.layer(x_h, r_h, dl.router_w_host, dl.bias_host, gc, gs, dc, ds, shared[0], shared[1],
                     cfg.top_k, experts=sel, n_threads=threads)
        spent += time.perf_counter() - t0
        nbytes += cfg.counted_bytes(len(sel))
        n += 1
    return {"value": round(nbytes / spent / 1e9, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} whole layer-step(s) of batch {B} (fp64 C++ oracle, OpenMP over {threads} threads), "
                      f"{spent:.1f} s", "us_per_step": round(spent / n * 1e6, 1)}


def main():
    args = parse_args()
    import synth
    cfg = synth.CONFIGS[args.config]
    if args.experts:
        cfg = cfg.with_(n_experts=args.experts, name=cfg.name + f"_E{args.experts}")
    global POOL
    POOL = args.pool
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
