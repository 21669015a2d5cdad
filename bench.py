#!/usr/bin/env python
"""Benchmark of the sparse MXFP4 MoE decode layer (libmoe_decode.so) on B200.

One step = one moe_layer_forward of the workload (router GEMV + top-k +
bucketing, routed MXFP4 SwiGLU experts, the shared expert, down projection
fused with the combine and residual add) on one batch of
seeded synthetic tokens; a pool of distinct tokens makes every step route to
a different expert set.  Weights and inputs are resident in HBM before the
timed region; L2 is flushed (256 MiB write) between steps, outside the
per-step CUDA events.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1|2|3|5] [--impl ours|reference]

With the default workload (the full-size batch-1 layer) on one GPU the line
also carries `per_config`: the batch-8, batch-64 (Zipf) and speculative
verify (8 correlated positions of one sequence) layers through the same
call, and the 4-layer x 64-step decode loop captured in one CUDA graph with
and without the next-layer L2 prefetch.

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
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the batch-8, batch-64 and 4-layer graph records of the default run")
    ap.add_argument("--flags", type=int, default=0, help="MOE_FLAG_* bits for ablations")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling aid: fewer routed experts (same per-step work, smaller footprint)")
    ap.add_argument("--pool", type=int, default=64, help="distinct token batches cycled through the steps")
    return ap.parse_args()


def workload_desc(cfg):
    return (f"{cfg.name}: one MoE decode layer, hidden {cfg.hidden}, {cfg.n_experts} routed experts top-{cfg.top_k}, "
            f"expert intermediate {cfg.inter} (MXFP4 E2M1 + E8M0/32), shared expert intermediate "
            f"{cfg.shared_inter} (bf16), batch {cfg.batch}" + (f", Zipf({cfg.zipf_s}) router bias" if cfg.zipf_s else ""))


def config_dict(cfg, world, flags):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": workload_desc(cfg), "batch": cfg.batch, "parallelism": f"replicas x{world}",
            "l2": "flushed between steps (256 MiB write, outside the per-step CUDA events)",
            "token_pool": POOL, "flags": flags}


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
    for f in ("kernels.cuh", "gemv.cuh", "ptx.cuh", "moe_decode.cu", "mx_umma.cuh", "persistent.cuh",
              "mma_grouped.cuh"):
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
            "config": config_dict(cfg, 1, args.flags),
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


class LayerRun:
    """One full-size layer on the device with a pool of distinct token
    batches, timed through moe_layer_forward (weights and inputs resident in
    HBM, L2 flushed between steps outside the per-step events)."""

    def __init__(self, cfg, flags, pool, layer=0):
        import torch
        from sparse_moe_decode_router_b200 import api
        from synth.workload import make_device_layer, residual_tokens
        self.torch, self.api, self.cfg = torch, api, cfg
        B, H = cfg.batch, cfg.hidden
        self.dl = make_device_layer(cfg, layer)
        c = api.moe_layer_config(cfg.hidden, cfg.n_experts, cfg.top_k, cfg.inter, cfg.shared_inter, B, flags)
        self.handle = api.moe_layer_create(c, self.dl.weights_struct())
        self.path = api.moe_layer_expert_path(self.handle, B)   # MOE_PATH_* of the routed experts
        self.pool = pool
        self.x, self.r, self.xh, self.rh = [], [], [], []
        for p in range(pool):
            ids = [p * B + b for b in range(B)]
            xh, xd = self.dl.tokens(ids)
            rh, rd = residual_tokens(cfg, ids)
            self.x.append(xd)
            self.r.append(rd)
            self.xh.append(torch.from_numpy(xh.view(np.int16)).pin_memory())
            self.rh.append(torch.from_numpy(rh.view(np.int16)).pin_memory())
        self.out = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        self.out_h = torch.empty((B, H), dtype=torch.int16).pin_memory()
        self.flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.stream = torch.cuda.current_stream()
        plan = api.moe_layer_routing(self.handle)
        n_act_view = torch.as_tensor(_DevPtr(plan.n_active, (1,), "<i4"), device="cuda")
        self.n_active = []
        for p in range(pool):           # experts touched by each pool batch (read back before timing)
            api.moe_layer_forward(self.handle, None, self.x[p], self.r[p], self.out, B, self.stream)
            self.n_active.append(int(n_act_view.cpu()[0]))
        torch.cuda.synchronize()
        if api.moe_layer_last_device_error(self.handle) != api.MOE_OK:
            raise SystemExit("device-side error during warm-up")

    def step_bytes(self, i):
        return self.cfg.counted_bytes(self.n_active[i % self.pool])

    def gate_up_bytes(self, i):
        """Routed gate/up kernel: codes + scales of the active experts, x in, h out (fp32)."""
        c = self.cfg
        na = self.n_active[i % self.pool]
        return na * 2 * c.inter * (c.hidden // 2 + c.hidden // 32) + c.batch * c.hidden * 2 + \
            c.batch * c.top_k * c.inter * 4

    def forward(self, i):
        self.api.moe_layer_forward(self.handle, None, self.x[i % self.pool], self.r[i % self.pool], self.out,
                                   self.cfg.batch, self.stream)

    def timed(self, steps, warmup, sampler=None, probe=False, host=False):
        """Per-step device times (ms) of `steps` steps after `warmup` untimed
        ones; probe: the routed gate/up kernel's own time instead."""
        torch, api = self.torch, self.api
        B = self.cfg.batch
        for i in range(warmup):
            self.flush.zero_()
            self.forward(i)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        if probe:
            for a, b in ev:  # materialise the events before handing them to the library
                a.record(self.stream)
                b.record(self.stream)
        torch.cuda.synchronize()
        if sampler:
            sampler.begin()
        for i in range(steps):
            self.flush.zero_()
            if probe:
                api.moe_layer_set_probe(self.handle, ev[i][0], ev[i][1])
                self.forward(i)
            elif host:
                ev[i][0].record(self.stream)
                api.moe_layer_forward_host(self.handle, self.xh[i % self.pool], self.rh[i % self.pool], self.out_h,
                                           B, self.stream)
                ev[i][1].record(self.stream)
            else:
                ev[i][0].record(self.stream)
                self.forward(i)
                ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        if sampler:
            sampler.end()
        if probe:
            api.moe_layer_set_probe(self.handle, None, None)
        if api.moe_layer_last_device_error(self.handle) != api.MOE_OK:
            raise SystemExit("device-side error during the timed region")
        return [a.elapsed_time(b) for a, b in ev]

    def close(self):
        self.api.moe_layer_destroy(self.handle)
        del self.dl, self.x, self.r, self.flush
        self.torch.cuda.empty_cache()


def grouped_flops(cfg, n_pairs):
    """Multiply-add work of the routed experts at one token per pair: gate/up
    (2I x H) and down (H x I) per pair, 2 flops per multiply-add."""
    return n_pairs * 2 * (2 * cfg.inter * cfg.hidden + cfg.hidden * cfg.inter)


def per_config_record(cfg, flags, steps, warmup, peak, sampler):
    from sparse_moe_decode_router_b200 import api
    persistent = bool(flags & api.MOE_FLAG_PERSISTENT) and cfg.batch == 1  # one cooperative launch
    run = LayerRun(cfg, flags, pool=8)
    try:
        ms = run.timed(steps, warmup, sampler)
        tot = sum(run.step_bytes(i) for i in range(steps))
        sec = sum(ms) * 1e-3
        rec = {"workload": workload_desc(cfg), "batch": cfg.batch, "steps": steps, "warmup": warmup,
               "us_per_step": round(sum(ms) / steps * 1e3, 2), "gb_per_s": round(tot / sec / 1e9, 2),
               "frac_of_measured_hbm": round(tot / sec / 1e9 / peak, 4),
               "tokens_per_s": round(cfg.batch * steps / sec, 1),
               "counted_bytes_per_step": int(tot / steps),
               "n_active_mean": statistics.mean(run.n_active[i % run.pool] for i in range(steps)),
               "gpu_launches_per_step": (1 if persistent else launches_per_step(cfg, run.path)),
               "expert_path": PATH_NAMES[run.path]}
        if run.path != 0:
            fl = grouped_flops(cfg, cfg.batch * cfg.top_k)
            rec["routed_tflops"] = round(fl * steps / sec / 1e12, 2)
        return rec
    finally:
        run.close()


def stack_record(cfg, flags, replays, peak, sampler):
    """Config 4: n_layers full-size layers chained through the residual, an
    n_steps decode loop captured in one CUDA graph (PDL inside, next-layer L2
    prefetch unless MOE_FLAG_NO_PREFETCH); device time per replay / layer-steps.
    Weights (~84 GB) exceed L2 many times over, so L2 is not flushed."""
    import torch
    from sparse_moe_decode_router_b200 import api
    from synth.workload import make_device_layer, residual_tokens
    nl, ns, H = cfg.n_layers, cfg.n_steps, cfg.hidden
    layers = [make_device_layer(cfg, l) for l in range(nl)]
    xs = [[None] * nl for _ in range(ns)]
    for l in range(nl):
        _, xd = layers[l].tokens(range(ns))
        for t in range(ns):
            xs[t][l] = xd[t:t + 1]
    _, r0 = residual_tokens(cfg, range(ns), 0)
    c = api.moe_layer_config(cfg.hidden, cfg.n_experts, cfg.top_k, cfg.inter, cfg.shared_inter, 1, flags)
    handles = [api.moe_layer_create(c, dl.weights_struct()) for dl in layers]
    try:
        outs = [[torch.empty((1, H), dtype=torch.bfloat16, device="cuda") for _ in range(nl)] for _ in range(ns)]
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for t in range(ns):
                    res = r0[t:t + 1]
                    for l in range(nl):
                        api.moe_layer_forward(handles[l], handles[(l + 1) % nl], xs[t][l], res, outs[t][l], 1,
                                              stream=torch.cuda.current_stream())
                        res = outs[t][l]
        st = torch.cuda.current_stream()
        g.replay()                      # warm-up
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
        sampler.begin()
        for a, b in ev:
            a.record(st)
            g.replay()
            b.record(st)
        torch.cuda.synchronize()
        sampler.end()
        for hd in handles:
            if api.moe_layer_last_device_error(hd) != api.MOE_OK:
                raise SystemExit("device-side error in the stack graph")
        del g
        ms = statistics.median(a.elapsed_time(b) for a, b in ev)
        per = ms * 1e3 / (nl * ns)
        bpl = cfg.counted_bytes(cfg.top_k)       # batch 1: top_k distinct experts per layer-step
        return {"us_per_layer_step": round(per, 2), "gb_per_s": round(bpl / (per * 1e-6) / 1e9, 2),
                "frac_of_measured_hbm": round(bpl / (per * 1e-6) / 1e9 / peak, 4),
                "replays": replays, "replay_ms_median": round(ms, 3), "layer_steps_per_replay": nl * ns,
                "gpu_launches_per_layer_step": launches_per_step(cfg.with_(batch=1),
                                                                 api.moe_layer_expert_path(handles[0], 1))}
    finally:
        for hd in handles:
            api.moe_layer_destroy(hd)
        del layers, xs
        torch.cuda.empty_cache()


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
    import synth

    api.load_library()
    B, H, k = cfg.batch, cfg.hidden, cfg.top_k
    run = LayerRun(cfg, args.flags, POOL)
    path = run.path
    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(local, uuid)
    sampler.start()
    K = args.steps
    # headline: whole layer-steps, nothing but the layer between the events
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = run.timed(K, args.warmup, sampler)
    if dist is not None:
        dist.barrier()
    # end to end through the host-buffer entry point (pinned host memory)
    e2e_ms = run.timed(K, min(args.warmup, 3), sampler, host=True)
    # the dominant kernel, timed live in a separate pass (events around it)
    gu_ms = run.timed(min(K, 100), 3, None, probe=True)
    total_ms = sum(step_ms)
    total_bytes = sum(run.step_bytes(i) for i in range(K))
    e2e_total = sum(e2e_ms)
    gu_avg_s = statistics.mean(gu_ms) * 1e-3
    gu_bytes = statistics.mean([run.gate_up_bytes(i) for i in range(len(gu_ms))])
    n_active_mean = statistics.mean(run.n_active[i % POOL] for i in range(K))
    if dist is not None:
        total_ms, e2e_total = max_over_ranks([total_ms, e2e_total], "cuda")
    peak, peak_src = measured_peaks()
    extra = {}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        extra["cpu_baseline"] = cpu_baseline(cfg, run.dl)
    run.close()
    if world == 1 and not args.no_per_config and cfg.name == synth.CONFIGS[1].name:
        extra["per_config"] = {
            "full_b8": per_config_record(synth.CONFIGS[2], args.flags, 50, 5, peak, sampler),
            "full_b64_zipf": per_config_record(synth.CONFIGS[3], args.flags, 20, 3, peak, sampler),
            "full_b8_verify": per_config_record(synth.CONFIGS[5], args.flags, 50, 5, peak, sampler),
            # batch-1 variants beside the default chain: the persistent single
            # launch, and the routed experts on the tensor cores
            "full_b1_persistent": per_config_record(synth.CONFIGS[1], args.flags | api.MOE_FLAG_PERSISTENT, 50, 5,
                                                    peak, sampler),
            "full_b1_tcgen05": per_config_record(synth.CONFIGS[1], args.flags | api.MOE_FLAG_MX_EXPERTS, 50, 5,
                                                 peak, sampler),
            "full_stack4_b1_graph": {
                "prefetch": stack_record(synth.CONFIGS[4], args.flags, 3, peak, sampler),
                "no_prefetch": stack_record(synth.CONFIGS[4], args.flags | api.MOE_FLAG_NO_PREFETCH, 3, peak,
                                            sampler)},
        }
    clocks = sampler.stop()
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_per_step = total_ms / K
    value = job_value(world, total_bytes, total_ms)
    achieved = gu_bytes / gu_avg_s / 1e9
    from sparse_moe_decode_router_b200.api import MOE_PATH_TCGEN05
    gu_tag = "routed_gate_up_tcgen05" if path == MOE_PATH_TCGEN05 else "routed_gate_up"
    traffic = recorded_traffic(gu_tag, cfg.name)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded Philox4x32-10 draws; random-init weights of the full-size layer)",
        "config": config_dict(cfg, world, args.flags),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "tokens_per_s": round(world * B * K / (total_ms * 1e-3), 1),
        "counted_bytes_per_step": int(total_bytes / K),
        "n_active_mean": n_active_mean,
        "frac_of_measured_hbm": round(value / world / peak, 4),
        "roofline": {"kernel": gu_tag, "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": peak_src, "algorithmic_bytes_per_launch": int(gu_bytes),
                     "avg_launch_us": round(gu_avg_s * 1e6, 2),
                     "timing": "separate pass: events recorded around the kernel on its stream"},
        "e2e": {"value": round(world * total_bytes / (e2e_total * 1e-3) / 1e9, 2), "unit": UNIT,
                "h2d_bytes_per_step": 2 * B * H * 2, "d2h_bytes_per_step": B * H * 2,
                "us_per_step": round(e2e_total / K * 1e3, 2)},
        "gpu_launches": launches_per_step(cfg, path) * K,
        "clocks": clocks,
    }
    line.update(extra)
    print(json.dumps(line), flush=True)


PATH_NAMES = {0: "CUDA-core GEMV kernels", 1: "grouped warp-MMA kernels", 2: "tcgen05 block-scaled kernels"}


def launches_per_step(cfg, path):
    """Kernels of this library one moe_layer_forward launches: the router
    (whose last CTA selects the top-k and builds the buckets, and which also
    streams a bf16 shared expert's gate/up rows), the shared expert's down
    projection (an MXFP4 shared expert: its gate/up and down); then the routed
    experts on the kernels moe_layer_expert_path names (`path`): tcgen05 =
    the activation-term kernel, gate/up and down+combine; grouped warp-MMA =
    an activation-staging kernel and a grouped MMA kernel per projection,
    then the combine; GEMV = the streaming gate/up and down+combine.  Above
    batch 1 on the tcgen05 path the router and the bf16 shared expert run on
    the dense tensor-core kernels (the router's launch, the shared down's) and
    the routing finish is a launch of its own; above batch 2 the combine
    follows the tcgen05 down projection as a launch of its own.  Where the
    hidden size is a multiple of 256 the tcgen05 gate/up kernel writes h in
    fp32 and a small kernel makes its E2M1 terms (one launch more)."""
    n = 1
    if cfg.shared_inter > 0:
        n += 2 if cfg.shared_format == "mxfp4" else 1
    if path == 2 and cfg.batch > 1:
        n += 1
    if path == 2 and cfg.batch > 2:
        n += 1
    if path == 2 and cfg.hidden % 256 == 0:
        n += 1
    return n + {2: 3, 1: 5, 0: 2}[path]


def _oracle_step(cfg, dl, n, threads):
    import oracle
    from synth.workload import residual_tokens
    B = cfg.batch
    ids = [((n % POOL) * B) + b for b in range(B)]
    x_h, _ = dl.tokens(ids)
    r_h, _ = residual_tokens(cfg, ids)
    rt = oracle.routing(x_h, dl.router_w_host, dl.bias_host, cfg.top_k)
    sel = np.unique(rt["topk_idx"])
    gc, gs, dc, ds = dl.host_experts(sel)
    shared = dl.host_shared()
    t0 = time.perf_counter()
    oracle.layer(x_h, r_h, dl.router_w_host, dl.bias_host, gc, gs, dc, ds, shared[0], shared[1],
                 cfg.top_k, experts=sel, n_threads=threads)
    return time.perf_counter() - t0, cfg.counted_bytes(len(sel))


def cpu_baseline(cfg, dl):
    """The oracle as it stands on the host cores, on a bounded sample of the
    same workload: whole layer-steps with OpenMP over all host threads until
    ~10 s of CPU work (at least one), then one layer-step on one thread."""
    threads = os.cpu_count() or 1
    B = cfg.batch
    spent, n, nbytes = 0.0, 0, 0
    while n < 1 or (spent < 10.0 and n < 64):
        dt, nb = _oracle_step(cfg, dl, n, threads)
        spent += dt
        nbytes += nb
        n += 1
    dt1, nb1 = _oracle_step(cfg, dl, n, 1)
    return {"value": round(nbytes / spent / 1e9, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} whole layer-step(s) of batch {B} (fp64 C++ oracle, OpenMP over {threads} threads), "
                      f"{spent:.1f} s; then one layer-step on one thread",
            "us_per_step": round(spent / n * 1e6, 1),
            "single_thread": {"value": round(nb1 / dt1 / 1e9, 4), "unit": UNIT, "cores": 1,
                              "us_per_step": round(dt1 * 1e6, 1)}}


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
