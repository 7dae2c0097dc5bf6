"""Throughput of causal attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = forward + backward (forge_attn_fwd, then forge_attn_bwd's three
stages) over one batch of the workload, inputs resident in HBM. The metric is
TFLOPS counting only causal / in-window score pairs: forward 4*D*pairs, backward
10*D*pairs (five D-deep products per pair, the recompute of S included).

N > 1 (torchrun, one process per GPU): every rank runs its own copy of the
workload (independent batches, no collective on the data path: weak scaling);
time is the max over ranks of the device-timed region.

--impl reference times the f64 CPU oracle on the host cores on a bounded sample
of the same workload (rank 0 only), in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1000 * 1000
METRIC = "causal attention fwd+bwd TFLOPS on 1 B200 and % of dense BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def flops_of(w):
    from causal_flash_attention_attn_b200.inputs import allowed_pairs
    pairs = allowed_pairs(w.T, w.window) * w.B * w.Hq
    return 4.0 * w.D * pairs, 10.0 * w.D * pairs


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def _strip_comments(text):
    """C/C++ source without // and /* */ comments (string literals kept), so that
    the hash below changes with the code and not with its comments."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join(out)


# The sources each captured kernel is built from: its own header(s) and the
# shared instruction wrappers. A traffic figure stands only while these are
# unchanged (the launch configuration lives beside the kernel, in its traits).
KERNEL_SOURCES = {
    "bwd_tc_kernel": ("bwd_tc.cuh", "sm100.cuh"),
    "fwd2_tc_kernel": ("fwd2_tc.cuh", "fwd_tc.cuh", "sm100.cuh"),
    "fwd_tc_kernel": ("fwd_tc.cuh", "sm100.cuh"),
    "decode_split": ("decode.cuh", "sm100.cuh"),
    "decode_split_warp": ("decode.cuh", "sm100.cuh"),
    "bwd_dkdv_tc_kernel": ("bwd_dkv.cuh", "bwd_tc.cuh", "fwd_tc.cuh", "sm100.cuh"),
    "bwd_dq_tc_kernel": ("bwd_dkv.cuh", "bwd_tc.cuh", "fwd_tc.cuh", "sm100.cuh"),
}


def kernel_source_hash(kernel=None):
    """sha256 prefix of the kernel's sources (all of csrc/ when kernel is None or
    unknown) without comments, whitespace runs collapsed (layout and comment edits
    leave it unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_flash_attention_attn_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    for name in sorted(names):
        with open(os.path.join(csrc, name), "r", encoding="utf-8") as f:
            h.update(name.encode())
            h.update(" ".join(_strip_comments(f.read()).split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when the summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def parse_smi_lines(lines):
    """(sm MHz samples, max MHz, reasons seen active) from nvidia-smi CSV lines of
    ClockSampler.SMI_FIELDS (noheader, nounits)."""
    sm, mx, reasons = [], None, set()
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for n, v in zip(REASON_NAMES, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return sm, mx, reasons


class ClockSampler:
    """SM clock and clock-event reasons of the GPU a run uses, sampled while its
    timed region runs (read-only: nothing here changes a GPU setting).

    NVML first: a thread reads the clock and the reasons every `period_s`, the GPU
    found by its UUID (then its PCI address) so that the sampled GPU is the one
    CUDA runs on; only samples between begin() and end() -- host times that
    bracket the timed region -- count. If NVML is unavailable, nvidia-smi polls
    every 100 ms and every sample counts."""
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_s=0.002):
        self.index = index
        self.period_s = period_s
        self.proc = None
        self.lines = []
        self.samples = []          # (host time, sm MHz, reason mask) from NVML
        self.t_begin = self.t_end = None
        self.nvml = None
        self.handle = None
        self.max_mhz = None
        self.bits = {}
        self.stop_evt = threading.Event()
        self.thread = None

    def _uuid(self):
        """NVML's name of the device ("GPU-" + 8-4-4-4-12 hex), or None."""
        import torch
        u = str(torch.cuda.get_device_properties(self.index).uuid)
        return "GPU-" + u if re.fullmatch(r"[0-9a-fA-F]{8}(-[0-9a-fA-F]{4}){3}-[0-9a-fA-F]{12}", u) else None

    # -- NVML
    def _nvml_handle(self, nv):
        import torch
        uuid = self._uuid()
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                pass
        props = torch.cuda.get_device_properties(self.index)
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        return nv.nvmlDeviceGetHandleByPciBusId(bus)

    def _start_nvml(self):
        import pynvml as nv
        nv.nvmlInit()
        try:
            self.handle = self._nvml_handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
            get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            for name, suffix in zip(REASON_NAMES, ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown",
                                                   "SwPowerCap")):
                self.bits[name] = getattr(nv, "nvmlClocksEventReason" + suffix,
                                          getattr(nv, "nvmlClocksThrottleReason" + suffix, 0))
            # one read before the thread starts, so a failing call falls back here
            nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            get(self.handle)
        except Exception:
            nv.nvmlShutdown()
            raise
        self.nvml = nv

        def loop():
            while not self.stop_evt.is_set():
                t = time.perf_counter()
                try:
                    mhz = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                    mask = int(get(self.handle))
                    self.samples.append((t, mhz, mask))
                except Exception:
                    pass
                self.stop_evt.wait(self.period_s)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    # -- nvidia-smi fallback
    def _start_smi(self):
        ident = str(self.index)
        try:
            ident = self._uuid() or ident
        except Exception:
            pass
        self.proc = subprocess.Popen(
            ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits",
             "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

        def read():
            for line in self.proc.stdout:
                self.lines.append(line.strip())

        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def start(self):
        try:
            self._start_nvml()
            return
        except Exception:
            self.nvml = None
        try:
            self._start_smi()
        except Exception:
            self.proc = None

    def begin(self):
        self.t_begin = time.perf_counter()

    def end(self):
        self.t_end = time.perf_counter()

    def stop(self):
        if self.nvml is not None:
            self.stop_evt.set()
            self.thread.join(timeout=2)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return self.summary_nvml()
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = parse_smi_lines(self.lines)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi every 100 ms (before, during and after the timed region)"}

    def summary_nvml(self):
        lo = self.t_begin if self.t_begin is not None else float("-inf")
        hi = self.t_end if self.t_end is not None else float("inf")
        inside = [(mhz, mask) for t, mhz, mask in self.samples if lo <= t <= hi]
        where = "inside the timed region"
        if not inside:
            # a region shorter than the period: the first sample after it began
            after = [(mhz, mask) for t, mhz, mask in self.samples if t >= lo]
            inside, where = after[:1], "first sample after the timed region began"
        if not inside:
            inside, where = [(mhz, mask) for _, mhz, mask in self.samples], "all samples (none after the region began)"
        if not inside:
            return None
        reasons = sorted(n for n in REASON_NAMES if any(mask & self.bits.get(n, 0) for _, mask in inside))
        return {"sm_mhz": statistics.median(m for m, _ in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside),
                "source": f"NVML every {self.period_s * 1e3:g} ms, {where}"}


# ------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity when world == 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank: float, max_ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling), the
    step time is the slowest rank's."""
    return world * flops_per_rank / (max_ms_per_step * 1e-3) / 1e12


def barrier(world: int, device=None):
    if world == 1:
        return
    import torch.distributed as dist
    if device is not None and device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


# ------------------------------------------------------------ CPU baseline
def _oracle_groups(w, groups, q, k, v, dO):
    """Seconds of the f64 oracle (fwd + bwd) over the listed (b, kv-head) groups."""
    import oracle
    G = w.G
    t0 = time.perf_counter()
    for b, h in groups:
        hs = slice(h * G, (h + 1) * G)
        ks, vs = k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1]
        qs, ds = q[b:b + 1, hs], dO[b:b + 1, hs]
        oracle.attn_fwd(qs, ks, vs, w.sm_scale, w.window, w.softcap)
        oracle.attn_bwd(qs, ks, vs, ds, w.sm_scale, w.window, w.softcap)
    return time.perf_counter() - t0


def cpu_oracle_sample(w, budget_s=12.0, max_groups=None):
    """Time the f64 oracle (fwd + bwd) on whole KV groups of the workload, adding
    groups until ~budget_s of CPU work. Returns (tflops, seconds, description, cores)."""
    import oracle
    from causal_flash_attention_attn_b200 import inputs
    from causal_flash_attention_attn_b200.inputs import allowed_pairs
    q, k, v, dO = inputs.make_inputs(w)
    groups = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    if max_groups:
        groups = groups[:max_groups]
    done, secs, flops = 0, 0.0, 0.0
    for g in groups:
        secs += _oracle_groups(w, [g], q, k, v, dO)
        flops += 14.0 * w.D * allowed_pairs(w.T, w.window) * w.G
        done += 1
        if secs >= budget_s:
            break
    desc = (f"f64 oracle fwd+bwd on {done} of {w.B * w.Hkv} KV groups (b, kv-head) of {w.name}, "
            f"each {w.G} query heads x T={w.T}")
    return flops / secs / 1e12, secs, desc, oracle.num_threads()


def cpu_oracle_full(names=("f32_correctness", "forge_default")):
    """The small workloads timed in full with the oracle's default threads, and the
    f32 correctness workload on one thread as well. Pairs per second count the
    allowed (query, key) pairs of the whole workload, forward and backward."""
    import oracle
    from causal_flash_attention_attn_b200 import inputs
    from causal_flash_attention_attn_b200.inputs import allowed_pairs
    out = {}
    for name in names:
        w = inputs.WORKLOADS[name]
        q, k, v, dO = inputs.make_inputs(w)
        groups = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
        pairs = allowed_pairs(w.T, w.window) * w.B * w.Hq
        secs = _oracle_groups(w, groups, q, k, v, dO)
        out[name] = {"seconds": round(secs, 4), "pairs_per_s": round(pairs / secs, 1),
                     "tflops": round(14.0 * w.D * pairs / secs / 1e12, 6), "threads": oracle.num_threads()}
    w = inputs.WORKLOADS["f32_correctness"]
    q, k, v, dO = inputs.make_inputs(w)
    before = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        secs = _oracle_groups(w, [(b, h) for b in range(w.B) for h in range(w.Hkv)], q, k, v, dO)
    finally:
        oracle.set_num_threads(before)
    pairs = allowed_pairs(w.T, w.window) * w.B * w.Hq
    out["f32_correctness_single_thread"] = {"seconds": round(secs, 4), "pairs_per_s": round(pairs / secs, 1),
                                            "tflops": round(14.0 * w.D * pairs / secs / 1e12, 6), "threads": 1}
    return out


# -------------------------------------------------------------------- ours
def spread(xs):
    """Median and spread of a list of per-step times (ms)."""
    ys = sorted(xs)
    n = len(ys)

    def pct(p):
        return ys[min(n - 1, max(0, int(round(p * (n - 1)))))]
    return {"median": round(statistics.median(ys), 4), "min": round(ys[0], 4), "p10": round(pct(0.1), 4),
            "p90": round(pct(0.9), 4), "max": round(ys[-1], 4), "n": n}


class Runner:
    """Device buffers and the timed step (forward, then the backward's three
    stages) of one workload on one GPU, through the library's C ABI."""

    def __init__(self, w, dev, stream, host_inputs=None):
        import torch
        import causal_flash_attention_attn_b200 as fa
        from causal_flash_attention_attn_b200 import inputs
        self.fa, self.w, self.dev, self.stream = fa, w, dev, stream
        self.host = host_inputs if host_inputs is not None else inputs.make_inputs(w)
        q, k, v, dO = self.host
        B, Hq, Hkv, T, D = w.B, w.Hq, w.Hkv, w.T, w.D
        self.dt = fa.dtype_code(inputs.torch_dtype(w.dtype))
        self.qd, self.kd, self.vd, self.dOd = (x.to(dev) for x in (q, k, v, dO))
        self.o = torch.empty_like(self.qd)
        self.lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.qd), torch.empty_like(self.kd), torch.empty_like(self.vd)
        self.nws = fa.forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, self.dt)
        self.ws = torch.empty(self.nws, dtype=torch.uint8, device=dev)
        # Timing hygiene: when the per-step working set is not well above the L2
        # size, every step first overwrites a 256 MB scratch buffer (outside the
        # timed kernels) so that no step starts with the previous one's data in L2.
        self.working_set = sum(x.numel() * x.element_size() for x in
                               (self.qd, self.kd, self.vd, self.o, self.lse, self.dOd, self.dq, self.dk, self.dv,
                                self.ws))
        self.flush = self.working_set < 2 * L2_BYTES
        self.scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if self.flush else None

    def step(self, ev=None):
        """One forward + backward. ev: None, 2 events (the step's bounds only, so
        that consecutive kernels may overlap their launch) or 5 (between every
        stage, for the per-kernel breakdown)."""
        import torch
        fa, w, sh = self.fa, self.w, self.stream.cuda_stream
        B, Hq, Hkv, T, D = w.B, w.Hq, w.Hkv, w.T, w.D
        sc, W, C, dt, ws, nws = w.sm_scale, w.window, w.softcap, self.dt, self.ws, self.nws
        if self.flush:
            with torch.cuda.stream(self.stream):
                self.scratch.fill_(1)
        full = ev is not None and len(ev) == 5
        if ev:
            ev[0].record(self.stream)
        s = fa.forge_attn_fwd(self.qd, self.kd, self.vd, self.o, self.lse, B, Hq, Hkv, T, D, sc, W, C, dt, sh)
        if full:
            ev[1].record(self.stream)
        s |= fa.forge_attn_bwd_preprocess(self.o, self.dOd, B, Hq, Hkv, T, D, dt, ws, nws, sh)
        if full:
            ev[2].record(self.stream)
        s |= fa.forge_attn_bwd_main(self.qd, self.kd, self.vd, self.lse, self.dOd, self.dq, self.dk, self.dv, B, Hq,
                                    Hkv, T, D, sc, W, C, dt, ws, nws, sh)
        if full:
            ev[3].record(self.stream)
        s |= fa.forge_attn_bwd_finalize(self.dq, B, Hq, Hkv, T, D, dt, ws, nws, sh)
        if ev:
            ev[-1].record(self.stream)
        if s != fa.FORGE_OK:
            raise fa.ForgeError(s, "step")

    def warm(self, n):
        import torch
        with torch.cuda.stream(self.stream):
            for _ in range(n):
                self.step()
        torch.cuda.synchronize(self.dev)
        st = self.fa.forge_attn_check(self.stream.cuda_stream)
        if st != self.fa.FORGE_OK:
            raise self.fa.ForgeError(st, "warmup")

    @staticmethod
    def per_kernel(evs):
        per = {"fwd": [], "bwd_preprocess": [], "bwd_main": [], "bwd_finalize": [], "step": []}
        for e in evs:
            per["fwd"].append(e[0].elapsed_time(e[1]))
            per["bwd_preprocess"].append(e[1].elapsed_time(e[2]))
            per["bwd_main"].append(e[2].elapsed_time(e[3]))
            per["bwd_finalize"].append(e[3].elapsed_time(e[4]))
            per["step"].append(e[0].elapsed_time(e[4]))
        return per

    def timed(self, steps, per_kernel=True):
        """Per-step CUDA-event times (ms), steps back to back: of each stage
        (per_kernel) or of the whole step only ({"step": [...]})."""
        import torch
        n = 5 if per_kernel else 2
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n)] for _ in range(steps)]
        for i in range(steps):
            self.step(evs[i])
        torch.cuda.synchronize(self.dev)
        st = self.fa.forge_attn_check(self.stream.cuda_stream)
        if st != self.fa.FORGE_OK:
            raise self.fa.ForgeError(st, "timed run")
        if per_kernel:
            return self.per_kernel(evs)
        return {"step": [e[0].elapsed_time(e[1]) for e in evs]}


def peak_for(kind, timed_s):
    peaks, src = load_peaks()
    key = kind + ("_sustained" if kind == "bf16_tflops" and timed_s > 2.0 else "")
    return float(peaks.get(key, FALLBACK_PEAKS[key])), f"{src} {key}"


def per_workload_block(args, dev, stream):
    """Every bf16 layer type of the workloads timed on its own (W untimed, then
    max(K, 30) timed steps; medians), plus the means the configurations pair the
    layer types into: the 16K model's 6-layer period (five W = 1024 layers, one
    global) and the Gemma-2-style 8K pair (one W = 4096 layer, one global)."""
    import torch
    from causal_flash_attention_attn_b200 import inputs
    out, cache = {}, {}
    steps = max(args.steps, 30)
    for name, w in inputs.WORKLOADS.items():
        if w.dtype != "bf16":
            continue
        key = (w.B, w.Hq, w.Hkv, w.T, w.D, w.seed, w.sigma_q, w.sigma_k, w.sigma_v, w.sigma_do)
        if key not in cache:
            cache.clear()
            cache[key] = inputs.make_inputs(w)
        r = Runner(w, dev, stream, host_inputs=cache[key])
        r.warm(args.warmup)
        with torch.cuda.stream(stream):
            whole = r.timed(steps, per_kernel=False)  # step times, nothing between the kernels
            per = r.timed(steps)                       # the per-stage breakdown
        fl_f, fl_b = flops_of(w)
        med = {k_: statistics.median(v_) for k_, v_ in per.items()}
        med["step"] = statistics.median(whole["step"])
        peak, _ = peak_for("bf16_tflops", sum(whole["step"]) * 1e-3)
        tf = (fl_f + fl_b) / (med["step"] * 1e-3) / 1e12
        out[name] = {"ms_step": round(med["step"], 4), "ms_step_sum_of_stages": round(statistics.median(per["step"]), 4),
                     "ms_fwd": round(med["fwd"], 4),
                     "ms_bwd_main": round(med["bwd_main"], 4),
                     "ms_bwd_pre_fin": round(med["bwd_preprocess"] + med["bwd_finalize"], 4),
                     "tflops": round(tf, 2), "frac": round(tf / peak, 4),
                     "fwd_frac": round(fl_f / (med["fwd"] * 1e-3) / 1e12 / peak, 4),
                     "bwd_main_frac": round(fl_b / (med["bwd_main"] * 1e-3) / 1e12 / peak, 4),
                     "gflop": round((fl_f + fl_b) / 1e9, 2), "l2_flushed": r.flush, "steps": steps}
        del r
        torch.cuda.empty_cache()
    peak, src = peak_for("bf16_tflops", 0.0)

    def mean(parts):
        ms = sum(n * out[k_]["ms_step"] for k_, n in parts)
        gf = sum(n * out[k_]["gflop"] for k_, n in parts)
        tf = gf / ms  # GFLOP / ms = TFLOP/s
        return {"layers": {k_: n for k_, n in parts}, "ms": round(ms, 4), "tflops": round(tf, 2),
                "frac": round(tf / peak, 4)}
    means = {}
    if "swa_w1024_16k" in out and "global_16k" in out:
        means["sliding_16k_period6 (5 x W1024 + 1 global)"] = mean([("swa_w1024_16k", 5), ("global_16k", 1)])
    if "softcap_w4096_8k" in out and "softcap_global_8k" in out:
        means["softcap_8k_alternating (1 x W4096 + 1 global)"] = mean([("softcap_w4096_8k", 1),
                                                                      ("softcap_global_8k", 1)])
    return {"layer_types": out, "means": means, "peak": peak, "peak_source": src,
            "timing": "per layer type: CUDA events around each stage, median of the timed steps; "
                      "step = fwd + bwd preprocess + bwd main + bwd finalize"}


def run_ours(args, w):
    import torch
    import causal_flash_attention_attn_b200 as fa

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.library()
    stream = torch.cuda.Stream(device=dev)

    # inputs: each rank its own batch of the workload (seed offset by rank)
    wr = w.with_(seed=w.seed + 1000 * rank) if rank else w
    r = Runner(wr, dev, stream)
    launches_per_step = 4
    r.warm(args.warmup)

    # the timed steps carry events at their bounds only (nothing between the
    # kernels of a step); the per-kernel breakdown is taken on K more steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clk = ClockSampler(dev.index)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    clk.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clk.begin()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            r.step(evs[i])
        end.record(stream)
    torch.cuda.synchronize(dev)
    clk.end()
    clocks = clk.stop()
    barrier(world, dev)
    st = fa.forge_attn_check(stream.cuda_stream)
    if st != fa.FORGE_OK:
        raise fa.ForgeError(st, "timed run")
    ms_local = start.elapsed_time(end)
    if r.flush:
        # the flushes sit between the timed kernels: time the kernels only
        ms_local = sum(e[0].elapsed_time(e[1]) for e in evs)
    ms = max_over_ranks(ms_local, world, dev)
    step_times = [e[0].elapsed_time(e[1]) for e in evs]
    with torch.cuda.stream(stream):
        per = r.timed(args.steps)
    avg = {kname: sum(v) / len(v) for kname, v in per.items() if kname != "step"}

    # end to end through the same C ABI from pinned host buffers: every step copies
    # its inputs host -> device and its gradients device -> host. The copies run on
    # their own streams into two alternating device buffer sets, so step k's
    # uploads overlap step k - 1's compute and downloads (PCIe carries both
    # directions at once); events order each buffer set's reuse.
    e2e = None
    if not args.no_e2e:
        q, k, v, dO = r.host
        hq_, hk_, hv_, hdo = (x.pin_memory() for x in (q, k, v, dO))
        hdq, hdk, hdv = (torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (r.qd, r.kd, r.vd))
        h2d = sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_, hdo))
        d2h = sum(x.numel() * x.element_size() for x in (hdq, hdk, hdv))
        bufs = [r, Runner(w, dev, stream, host_inputs=r.host)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def e2e_step(i):
            j, b = i % 2, bufs[i % 2]
            if used[j]:
                up.wait_event(comp_done[j])      # step i - 2 has read this set's inputs
            with torch.cuda.stream(up):
                for dst, src in ((b.qd, hq_), (b.kd, hk_), (b.vd, hv_), (b.dOd, hdo)):
                    dst.copy_(src, non_blocking=True)
                up_done[j].record(up)
            stream.wait_event(up_done[j])
            if used[j]:
                stream.wait_event(down_done[j])  # step i - 2's gradients are on the host
            with torch.cuda.stream(stream):
                b.step()
                comp_done[j].record(stream)
            down.wait_event(comp_done[j])
            with torch.cuda.stream(down):
                for dst, src in ((hdq, b.dq), (hdk, b.dk), (hdv, b.dv)):
                    dst.copy_(src, non_blocking=True)
                down_done[j].record(down)
            used[j] = True

        def e2e_run(n, s0=None, s1=None):
            if s0 is not None:
                s0.record(stream)
                up.wait_event(s0)
            for i in range(n):
                e2e_step(i)
            for j in range(2):
                if used[j]:
                    stream.wait_event(down_done[j])
            if s1 is not None:
                s1.record(stream)

        e2e_run(2)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        e2e_run(args.steps, s0, s1)
        torch.cuda.synchronize(dev)
        st = fa.forge_attn_check(stream.cuda_stream)
        if st != fa.FORGE_OK:
            raise fa.ForgeError(st, "end-to-end run")
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), world, dev) / args.steps
        fl_f, fl_b = flops_of(w)
        e2e = {"value": round(aggregate_tflops(world, fl_f + fl_b, e2e_ms), 3), "unit": "TFLOPS",
               "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": "pinned host, own H2D and D2H streams, two device buffer sets, overlapping compute"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return None

    fl_f, fl_b = flops_of(w)
    ms_step = ms / args.steps
    tflops = aggregate_tflops(world, fl_f + fl_b, ms_step)
    peak, peak_src = peak_for("bf16_tflops", ms * 1e-3)
    # dominant kernel: the larger of forward and backward-main by time
    dom = "bwd_main" if avg["bwd_main"] >= avg["fwd"] else "fwd"
    dom_flops = fl_b if dom == "bwd_main" else fl_f
    achieved = dom_flops / (avg[dom] * 1e-3) / 1e12
    kname = {"fwd": "fwd_tc_kernel" if w.D == 256 else "fwd2_tc_kernel", "bwd_main": "bwd_tc_kernel"}[dom]
    traffic = ncu_traffic(kname, w.name)
    line = {
        "metric": METRIC,
        "value": round(tflops, 3),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0, sigma^2) Q, K, V, dO)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "D": w.D,
                   "window": w.window, "softcap": w.softcap, "scale": w.sm_scale,
                   "parallelism": f"replicas x{world} (independent batches, no collective)",
                   "flops_per_step_per_gpu": fl_f + fl_b,
                   "flop_count": "only causal/in-window pairs; fwd 4*D*pairs, bwd 10*D*pairs",
                   "l2": ("flushed: a 256 MB buffer is written before each step (working set "
                          f"{r.working_set / 1e6:.0f} MB); step time = sum of the kernels' CUDA-event times")
                   if r.flush else
                   (f"not flushed: per-step working set (q,k,v,o,dO,dq,dk,dv,lse + workspace) "
                    f"{r.working_set / 1e6:.0f} MB exceeds twice the 126 MB L2")},
        "pct_of_bf16_peak": round(100.0 * tflops / world / peak, 2),
        "kernels_ms": {k_: round(v_, 4) for k_, v_ in avg.items()},
        "step_ms": spread(step_times),
        "kernels_ms_spread": {k_: spread(v_) for k_, v_ in per.items() if k_ != "step"},
        "roofline": {"kernel": kname, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": peak_src,
                     "achieved_def": f"{'10' if dom == 'bwd_main' else '4'}*D*pairs per launch / "
                                     "CUDA-event launch time (mean over the timed steps)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e:
        line["e2e"] = e2e
    del r
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_workload:
        line["per_workload"] = per_workload_block(args, dev, stream)
    if world == 1 and not args.no_cpu:
        v_, secs, desc, cores = cpu_oracle_sample(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(v_, 6), "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2),
                                "os_cpu_count": os.cpu_count(),
                                "OMP_NUM_THREADS": os.environ.get("OMP_NUM_THREADS"),
                                "full": cpu_oracle_full()}
    return line


def run_reference(args, w):
    """The oracle as it stands, on the host cores: W untimed then K timed steps,
    each step one bounded sample (one whole KV group of the workload, cycling
    through the groups)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    from causal_flash_attention_attn_b200 import inputs
    from causal_flash_attention_attn_b200.inputs import allowed_pairs
    q, k, v, dO = inputs.make_inputs(w)
    G = w.G
    groups = [(b, h) for b in range(w.B) for h in range(w.Hkv)]

    def sample(i):
        b, h = groups[i % len(groups)]
        hs = slice(h * G, (h + 1) * G)
        qs, ds = q[b:b + 1, hs], dO[b:b + 1, hs]
        ks, vs = k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1]
        t0 = time.perf_counter()
        oracle.attn_fwd(qs, ks, vs, w.sm_scale, w.window, w.softcap)
        oracle.attn_bwd(qs, ks, vs, ds, w.sm_scale, w.window, w.softcap)
        return time.perf_counter() - t0

    for i in range(args.warmup):
        sample(i)
    secs = sum(sample(i) for i in range(args.steps))
    flops = 14.0 * w.D * allowed_pairs(w.T, w.window) * G * args.steps
    value = flops / secs / 1e12
    fl_f, fl_b = flops_of(w)
    desc = (f"f64 oracle fwd+bwd, one KV group (b, kv-head: {G} query heads x T={w.T}) of {w.name} per step")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0, sigma^2) Q, K, V, dO)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "D": w.D,
                   "window": w.window, "softcap": w.softcap, "flops_per_step_full": fl_f + fl_b},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# KV-cache decode workload: a long-context batch, one new token per entry
DECODE = {"workload": "decode_b16_h32_kv8_t16k_d128", "B": 16, "Hq": 32, "Hkv": 8, "T": 16384, "Tmax": 16384,
          "D": 128, "dtype": "bf16", "window": 0, "softcap": 0.0}


def run_decode(args):
    """--decode: the KV-cache decode kernels (split + combine) on one GPU, HBM-bound:
    achieved = bytes of the K and V cache (plus q and o) per call / CUDA-event time."""
    import torch
    import causal_flash_attention_attn_b200 as fa

    c = DECODE
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fa.library()
    stream = torch.cuda.Stream(device=dev)
    g = torch.Generator(device="cpu").manual_seed(5)
    B, Hq, Hkv, T, Tmax, D = c["B"], c["Hq"], c["Hkv"], c["T"], c["Tmax"], c["D"]
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16).to(dev)
    kc = torch.randn(B, Hkv, Tmax, D, generator=g).to(torch.bfloat16).to(dev)
    vc = torch.randn(B, Hkv, Tmax, D, generator=g).to(torch.bfloat16).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    nws = fa.forge_attn_decode_workspace_size(B, Hq, Hkv, T, D)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    sc = 1.0 / math.sqrt(D)

    def call():
        s = fa.forge_attn_decode(q, kc, vc, o, lse, None, B, Hq, Hkv, T, Tmax, D, sc, c["window"], c["softcap"],
                                 None, fa.FORGE_DTYPE_BF16, ws, nws, stream.cuda_stream)
        if s != fa.FORGE_OK:
            raise fa.ForgeError(s, "decode")

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index)
    clk.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk.begin()
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk.end()
    clocks = clk.stop()
    st = fa.forge_attn_check(stream.cuda_stream)
    if st != fa.FORGE_OK:
        raise fa.ForgeError(st, "decode timed run")
    ms = e0.elapsed_time(e1) / args.steps
    cache_bytes = 2 * B * Hkv * T * D * 2
    io_bytes = 2 * B * Hq * D * 2 + B * Hq * 4
    gbs = (cache_bytes + io_bytes) / (ms * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"metric": "KV-cache decode bandwidth (one query per entry and head, K and V read once)",
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) q and caches)",
            "config": dict(c, l2="not flushed: the 1.07 GB cache exceeds the 126 MB L2"),
            "roofline": {"kernel": "decode_split_warp", "bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(gbs / peak, 4),
                         "traffic": ncu_traffic("decode_split_warp", c["workload"]),
                         "peak_source": f"{peak_src} hbm_gbs",
                         "achieved_def": "K+V cache bytes + q, o, lse bytes per call / CUDA-event time of both kernels"},
            "gpu_launches": 2 * args.steps, "clocks": clocks}


# d_k != d_v (decompressed multi-head latent attention) on the f32 CUDA-core path
DKV = {"workload": "mla_f32_b1_h16_t4096_dk192_dv128", "B": 1, "Hq": 16, "Hkv": 16, "T": 4096, "Dk": 192, "Dv": 128,
       "dtype": "f32", "window": 0, "softcap": 0.0}
# FP32 FMA peak of the CUDA cores: 148 SMs x 128 FMA lanes x 2 flops x 1.965 GHz
F32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_dkv(args):
    """--dkv: forward + backward with d_k = 192, d_v = 128 (f32, CUDA cores), FLOPs
    counted per allowed pair as 2 (Dk + Dv) forward and 2 (3 Dk + 2 Dv) backward
    (S recompute, dP, dV, dK, dQ), against the FP32 FMA peak."""
    import torch
    import causal_flash_attention_attn_b200 as fa

    c = DKV
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fa.library()
    stream = torch.cuda.Stream(device=dev)
    g = torch.Generator(device="cpu").manual_seed(6)
    B, Hq, Hkv, T, Dk, Dv = c["B"], c["Hq"], c["Hkv"], c["T"], c["Dk"], c["Dv"]
    q = torch.randn(B, Hq, T, Dk, generator=g).to(dev)
    k = torch.randn(B, Hkv, T, Dk, generator=g).to(dev)
    v = torch.randn(B, Hkv, T, Dv, generator=g).to(dev)
    dO = torch.randn(B, Hq, T, Dv, generator=g).to(dev)
    o = torch.empty(B, Hq, T, Dv, device=dev)
    lse = torch.empty(B, Hq, T, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nws = fa.forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, fa.FORGE_DTYPE_F32)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    sc = 1.0 / math.sqrt(Dk)
    sh = stream.cuda_stream

    def step():
        s = fa.forge_attn_fwd_dkv(q, k, v, o, lse, B, Hq, Hkv, T, Dk, Dv, sc, 0, 0.0, fa.FORGE_DTYPE_F32, sh)
        s |= fa.forge_attn_bwd_dkv(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, Dk, Dv, sc, 0, 0.0,
                                   fa.FORGE_DTYPE_F32, ws, nws, sh)
        if s != fa.FORGE_OK:
            raise fa.ForgeError(s, "dkv")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index)
    clk.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk.begin()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk.end()
    clocks = clk.stop()
    st = fa.forge_attn_check(sh)
    if st != fa.FORGE_OK:
        raise fa.ForgeError(st, "dkv timed run")
    ms = e0.elapsed_time(e1) / args.steps
    pairs = B * Hq * T * (T + 1) // 2
    flops = pairs * (2 * (Dk + Dv) + 2 * (3 * Dk + 2 * Dv))
    tf = flops / (ms * 1e-3) / 1e12
    return {"metric": "d_k != d_v attention fwd+bwd TFLOPS (f32 CUDA-core path)", "value": round(tf, 3),
            "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded N(0,1) q, k, v, dO)",
            "config": dict(c, l2="not flushed: the per-step working set (about 0.2 GB) exceeds the 126 MB L2",
                           flop_count="allowed pairs x (2 (Dk + Dv) forward + 2 (3 Dk + 2 Dv) backward)"),
            "roofline": {"kernel": "simt_bwd_dkdv", "bound": "alu", "achieved": round(tf, 3),
                         "peak": round(F32_FMA_TFLOPS, 1), "unit": "TFLOP/s", "frac": round(tf / F32_FMA_TFLOPS, 4),
                         "traffic": None, "peak_source": "148 SMs x 128 FP32 FMA lanes x 2 x 1.965 GHz",
                         "achieved_def": "all fwd+bwd flops / CUDA-event step time"},
            "gpu_launches": 4 * args.steps, "clocks": clocks}


# the same shapes in bf16 on the tensor cores; B = 4 so the working set (about
# 0.45 GB) exceeds the L2
DKV_BF16 = {"workload": "mla_bf16_b4_h16_t4096_dk192_dv128", "B": 4, "Hq": 16, "Hkv": 16, "T": 4096, "Dk": 192,
            "Dv": 128, "dtype": "bf16", "window": 0, "softcap": 0.0}


def run_dkv_bf16(args):
    """--dkv --dkv-dtype bf16: forward (fwd_tc_kernel<192, 128>) and backward
    (preprocess, bwd_dkdv_tc_kernel, bwd_dq_tc_kernel) on the tensor cores.
    FLOPs per allowed pair: 2 (Dk + Dv) forward, 2 (3 Dk + 2 Dv) backward (the
    algorithmic count; the two backward kernels recompute S and dP, which is not
    counted). Against the measured bf16 burst peak."""
    import torch
    import causal_flash_attention_attn_b200 as fa

    c = DKV_BF16
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fa.library()
    stream = torch.cuda.Stream(device=dev)
    g = torch.Generator(device="cpu").manual_seed(6)
    B, Hq, Hkv, T, Dk, Dv = c["B"], c["Hq"], c["Hkv"], c["T"], c["Dk"], c["Dv"]
    q = torch.randn(B, Hq, T, Dk, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(B, Hkv, T, Dk, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(B, Hkv, T, Dv, generator=g).to(torch.bfloat16).to(dev)
    dO = torch.randn(B, Hq, T, Dv, generator=g).to(torch.bfloat16).to(dev)
    o = torch.empty(B, Hq, T, Dv, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, Hq, T, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nws = fa.forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, fa.FORGE_DTYPE_BF16)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    sc = 1.0 / math.sqrt(Dk)
    sh = stream.cuda_stream

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        s = fa.forge_attn_fwd_dkv(q, k, v, o, lse, B, Hq, Hkv, T, Dk, Dv, sc, 0, 0.0, fa.FORGE_DTYPE_BF16, sh)
        if ev:
            ev[1].record(stream)
        s |= fa.forge_attn_bwd_dkv(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, Dk, Dv, sc, 0, 0.0,
                                   fa.FORGE_DTYPE_BF16, ws, nws, sh)
        if ev:
            ev[2].record(stream)
        if s != fa.FORGE_OK:
            raise fa.ForgeError(s, "dkv bf16")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clk = ClockSampler(dev.index)
    clk.start()
    time.sleep(0.3)
    clk.begin()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    clk.end()
    clocks = clk.stop()
    st = fa.forge_attn_check(sh)
    if st != fa.FORGE_OK:
        raise fa.ForgeError(st, "dkv bf16 timed run")
    fwd = [e[0].elapsed_time(e[1]) for e in evs]
    bwd = [e[1].elapsed_time(e[2]) for e in evs]
    ms = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    pairs = B * Hq * T * (T + 1) // 2
    fl_f, fl_b = pairs * 2 * (Dk + Dv), pairs * 2 * (3 * Dk + 2 * Dv)
    tf = (fl_f + fl_b) / (ms * 1e-3) / 1e12
    peak, peak_src = peak_for("bf16_tflops", 0.0)
    bwd_tf = fl_b / (statistics.median(bwd) * 1e-3) / 1e12
    return {"metric": "d_k != d_v attention fwd+bwd TFLOPS (bf16 tensor cores)", "value": round(tf, 3),
            "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "step_ms": spread([e[0].elapsed_time(e[2]) for e in evs]),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) q, k, v, dO)",
            "config": dict(c, l2="not flushed: the per-step working set (about 0.45 GB) exceeds the 126 MB L2",
                           flop_count="allowed pairs x (2 (Dk + Dv) forward + 2 (3 Dk + 2 Dv) backward)"),
            "kernels_ms": {"fwd": round(statistics.median(fwd), 4), "bwd": round(statistics.median(bwd), 4)},
            "pct_of_bf16_peak": round(100 * tf / peak, 2),
            "roofline": {"kernel": "bwd (preprocess + bwd_dkdv_tc_kernel + bwd_dq_tc_kernel)", "bound": "tensor",
                         "achieved": round(bwd_tf, 3), "peak": peak, "unit": "TFLOP/s", "frac": round(bwd_tf / peak, 4),
                         "traffic": None, "peak_source": peak_src,
                         "achieved_def": "2 (3 Dk + 2 Dv) flops per allowed pair / CUDA-event time of the backward call"},
            "gpu_launches": 4 * args.steps, "clocks": clocks}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-layer-type block (every bf16 workload timed on its own)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--decode", action="store_true", help="time the KV-cache decode kernels instead")
    ap.add_argument("--dkv", action="store_true", help="time the d_k != d_v path instead")
    ap.add_argument("--dkv-dtype", choices=["f32", "bf16"], default="f32",
                    help="f32: forward + backward on the CUDA cores; bf16: forward + backward on the tensor cores")
    args = ap.parse_args(argv)
    from causal_flash_attention_attn_b200 import inputs
    w = inputs.WORKLOADS[args.workload or inputs.HEADLINE]
    if args.warmup < 3:
        args.warmup = 3
    if args.decode:
        print(json.dumps(run_decode(args)), flush=True)
        return
    if args.dkv:
        print(json.dumps(run_dkv_bf16(args) if args.dkv_dtype == "bf16" else run_dkv(args)), flush=True)
        return
    line = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
