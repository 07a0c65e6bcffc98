#!/usr/bin/env python
"""Throughput of the top-k MoE FFN forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one whole forward (router, permutation, both grouped GEMMs,
combine) over one batch of synthetic tokens, through the C ABI.  The default
workload is the Mixtral-8x7B-shaped bf16 layer (T=4096 tokens, D=4096,
F=14336, E=8, top_k=2), the configuration the bf16-peak target is quoted on.
With N > 1 (torchrun) each rank runs an independent replica on its own GPU
(tokens are independent: no collective on the data path); the timing is the
max over ranks and ``value`` counts every rank's tokens.

Printed: one JSON line (rank 0) with tokens/s (``value``), routed TFLOP/s,
``roofline`` of the dominant kernel (timed live with CUDA events on the
launching stream), ``e2e`` (pinned host buffers, copies inside the timed
region), ``cpu_baseline`` (the float64 oracle on a bounded token sample on
this host's cores), ``clocks`` sampled through NVML during the timed region.

``--impl reference`` times the float64 oracle (the only reference this
subject has) on the same workload, on host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-FFN fwd tokens/s + routed TFLOP/s (% B200 bf16 peak; % HBM at small T)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
L2_BYTES = 126 * 1024 * 1024
# The configs timed after the headline one in the same run (each with its own
# inputs, warm-up, timed forwards and per-stage pass).
EXTRA_WORKLOADS = ("decode_t32_d4096_f14336_e8_k1_bf16", "decode_t32_d4096_f14336_e8_k2_bf16",
                   "decode_t32_d4096_f14336_e8_k8_bf16",
                   "fine_grained_t16384_d2048_f1408_e64_k6_zipf_bf16",
                   "dense_relu_t64_d32_f64_e4_k2_f32", "silu_gated_t64_d64_f128_e8_k2_f32")


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS)


KERNEL_SOURCES = {"gate_up": ("gemm_tc.cu", "common.cuh"),          # one CTA per tile
                  "gate_up_pair": ("gemm_tc2.cu", "common.cuh")}    # CTA pairs


def source_hash(kernel: str) -> str:
    """Hash of a grouped GEMM's sources: a stored DRAM-traffic figure is only
    reported while it matches the kernel it was taken on."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "mixture_experts_ffn_09_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str, kernel: str):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
        e = d[workload][kernel]
        if e.get("source_hash") == source_hash(kernel):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read only)."""

    NAMES = {"nvmlClocksEventReasonGpuIdle": "gpu_idle",
             "nvmlClocksEventReasonApplicationsClocksSetting": "applications_clocks_setting",
             "nvmlClocksEventReasonSwPowerCap": "sw_power_cap",
             "nvmlClocksEventReasonHwSlowdown": "hw_slowdown",
             "nvmlClocksEventReasonSyncBoost": "sync_boost",
             "nvmlClocksEventReasonSwThermalSlowdown": "sw_thermal_slowdown",
             "nvmlClocksEventReasonHwThermalSlowdown": "hw_thermal_slowdown",
             "nvmlClocksEventReasonHwPowerBrakeSlowdown": "hw_power_brake_slowdown",
             "nvmlClocksEventReasonDisplayClockSetting": "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01, pci_bus_id: str = None):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self.device_index = device_index
        self.pci_bus_id = pci_bus_id      # NVML numbers GPUs without CUDA_VISIBLE_DEVICES
        self._stop = threading.Event()
        self._ready = threading.Event()
        self.ok = False
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        # NVML is initialised and queried on this thread only: a driver call
        # that stalls can then never block the bench itself
        try:
            import pynvml as N
            N.nvmlInit()
            h = None
            if self.pci_bus_id:
                try:
                    h = N.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id)
                except Exception:
                    h = None
            if h is None:
                h = N.nvmlDeviceGetHandleByIndex(self.device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._ready.set()
        if not self.ok:
            return
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
                bits = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                for attr, name in self.NAMES.items():
                    v = getattr(N, attr, None)
                    if v is not None and bits & v:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self, wait_s: float = 5.0):
        """Starts sampling; waits at most ``wait_s`` for NVML to come up."""
        self.t.start()
        self._ready.wait(wait_s)

    def stop(self, wait_s: float = 2.0) -> dict:
        self._stop.set()
        self.t.join(wait_s)
        if self.t.is_alive() or not self.ok:
            why = "nvml stalled" if self.t.is_alive() else "nvml unavailable"
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [why],
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def cuda_pci_bus_id(index: int):
    """'DDDDDDDD:BB:DD.0' of a CUDA device, the form NVML looks GPUs up by."""
    try:
        import torch
        p = torch.cuda.get_device_properties(index)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ----------------------------------------------------------- accounting
def routed_flops(w, K=None) -> float:
    return w.routed_flops() if K is None else w.with_K(K).routed_flops()


def gate_up_flops(w) -> float:
    return float((4 if w.act == "silu_gated" else 2) * w.R * w.D * w.F)


def algorithmic_bytes(w, touched: int) -> float:
    """Weights of the experts actually selected, x in, out, selections and
    weights; the expert-sorted copies and intermediates are overhead."""
    s = 2 if w.dtype == "bf16" else 4
    gu_rows = 2 * w.F if w.act == "silu_gated" else w.F
    weights = touched * (gu_rows * w.D + w.D * w.F) * s + w.E * w.D * s
    return float(weights + 2 * w.T * w.D * s + w.T * w.K * 12)


def gate_up_bytes(w, touched: int) -> float:
    s = 2 if w.dtype == "bf16" else 4
    gu_rows = 2 * w.F if w.act == "silu_gated" else w.F
    return float(touched * gu_rows * w.D * s + w.R * w.D * s + w.R * w.F * s)


# ------------------------------------------------------------ oracle timing
def oracle_rate(w, d, budget_s: float, first_n: int = 8):
    """Tokens/s of the float64 oracle (dense over all experts, as it stands)
    on a bounded token sample.  Returns (tokens_per_s, n_tokens, seconds)."""
    import numpy as np
    from oracle import moe_oracle as O
    from mixture_experts_ffn_09_b200 import synth
    x = synth.as_float32(d["x"]).reshape(-1, w.D)
    gu = synth.as_float32(d["gate_up_proj"]).astype(np.float64)
    dn = synth.as_float32(d["down_proj"]).astype(np.float64)
    rt = synth.as_float32(d["router"]).astype(np.float64)

    def run(n):
        t0 = time.perf_counter()
        O.moe_ffn_forward(x[:n], rt, gu, dn, w.K, w.norm_topk_prob, w.act, d["router_bias"],
                          d["b1"], d["b2"])
        return time.perf_counter() - t0

    # a call has a large fixed cost (it streams every expert's float64
    # weights), so the sample grows until one call takes about the budget
    n = min(first_n, w.T)
    t = run(n)
    for _ in range(4):
        if t >= budget_s / 2 or n >= w.T:
            break
        n = int(min(w.T, max(2 * n, n * (budget_s / max(t, 1e-6)))))
        t = run(n)
    if t < budget_s / 2:
        # the whole batch is quick (the small layers): repeat it
        reps = int(min(10000, max(2, budget_s / 2 / max(t, 1e-6))))
        t = sum(run(n) for _ in range(reps))
        n *= reps
    return n / t, n, t


def oracle_rate_single_core(w, d, budget_s: float):
    """The same rate with the BLAS pool held to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return oracle_rate(w, d, budget_s)


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        nt = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if nt:
            return int(max(nt))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------- ranks
class Watchdog:
    """Bounded waits for the device work of one rank.

    Every point where the bench waits for the GPU goes through ``sync``: it
    records an event on the stream and polls it; work that has not finished
    after ``limit_s`` ends the process with a one-line error naming the phase
    (process exit tears the context down, so a stalled kernel cannot hold the
    GPU), instead of blocking until an outside timeout kills the job."""

    def __init__(self, dev, stream, limit_s: float):
        self.dev, self.stream, self.limit_s = dev, stream, limit_s

    def wait_event(self, ev, what: str):
        t0 = time.monotonic()
        while not ev.query():
            if time.monotonic() - t0 > self.limit_s:
                self.fail(what)
            time.sleep(0.0005)

    def fail(self, what: str):
        msg = {"error": f"device work of phase '{what}' did not finish within "
                        f"{self.limit_s:.0f} s"}
        try:
            from mixture_experts_ffn_09_b200 import moe
            word = moe.device_error_peek()
            msg["device_error_word"] = hex(word)
            msg["timed_out_in"] = moe.error_sites(word)
        except Exception as e:   # the report must not hang or raise
            msg["device_error_word"] = f"unreadable: {e}"
        print(json.dumps(msg), flush=True)
        os._exit(3)

    def sync(self, what: str):
        import torch
        ev = torch.cuda.Event()
        ev.record(self.stream)
        self.wait_event(ev, what)
        torch.cuda.synchronize(self.dev)

    def run(self, n: int, fn, what: str, chunk: int = 32):
        """Calls fn() n times, keeping the host at most two chunks of calls
        ahead of the device, so a stalled kernel is caught here rather than
        in a launch that blocks on a full queue."""
        import torch
        pending = []
        for i in range(n):
            fn()
            if (i + 1) % chunk == 0 or i + 1 == n:
                ev = torch.cuda.Event()
                ev.record(self.stream)
                pending.append((i, ev))
                if len(pending) > 2:
                    j, old = pending.pop(0)
                    self.wait_event(old, f"{what}, step {j}")


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (identity at world 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(local_ms_total: float, steps: int, tokens_per_rank: int, world: int, device=None):
    """(ms per step, whole-job tokens/s): the slowest rank's time over the
    tokens of every rank (weak scaling: each rank runs its own batch)."""
    ms = max_over_ranks(local_ms_total, world, device)
    ms_step = ms / max(steps, 1)
    return ms_step, world * tokens_per_rank / (ms_step / 1e3)


def init_dist(world: int, backend: str):
    if world <= 1:
        return
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def workload_config(w, world: int) -> dict:
    return {"workload": w.name, "T": w.T, "D": w.D, "F": w.F, "E": w.E, "K": w.K, "act": w.act,
            "norm_topk_prob": w.norm_topk_prob, "tokens_per_gpu": w.T,
            "global_batch_tokens": w.T * world,
            "parallelism": "replicas" if world > 1 else "single-gpu",
            "l2": "inputs larger than L2 (expert weights streamed every step)"
            if algorithmic_bytes(w, w.E) > L2_BYTES else "L2 not flushed (inputs fit in L2)"}


# ---------------------------------------------------------------- our arm
PEAK_FLOP_PER_CLK_PER_SM = 8192     # dense bf16 tcgen05 MMA: 8192 FLOP per SM per clock
SMS = 148
SUSTAINED_AFTER_S = 2.0             # a kernel timed inside a loop this long runs power-capped


def _readonly_view(a):
    """torch view of a read-only numpy array that is only ever read (copied
    to the device or to pinned memory), without torch's writability warning."""
    import warnings
    import numpy as np
    import torch
    with warnings.catch_warnings():
        warnings.filterwarnings("ignore", message="The given NumPy array is not writable")
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a))


class Layer:
    """Device buffers of one workload and the forward through the C ABI."""

    def __init__(self, w, d, dev, args, ext_opts=None):
        import torch
        from mixture_experts_ffn_09_b200 import moe
        self.w, self.dev = w, dev
        up = (lambda a: None if a is None else _readonly_view(a).to(dev))
        self.x = up(d["x"]).reshape(w.T, w.D)
        self.router, self.gu, self.dn = up(d["router"]), up(d["gate_up_proj"]), up(d["down_proj"])
        self.rb, self.b1, self.b2 = up(d["router_bias"]), up(d["b1"]), up(d["b2"])
        self.dt = moe.BF16 if w.dtype == "bf16" else moe.F32
        self.act = moe.ACT_NAMES[w.act]
        self.ws = torch.empty(moe.workspace_size(w.T, w.D, w.F, w.E, w.K, self.dt, self.act),
                              dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(self.x)
        self.sel = torch.empty(w.T, w.K, dtype=torch.int64, device=dev)
        self.wts = torch.empty(w.T, w.K, dtype=torch.float32, device=dev)
        self.ext = ext_opts
        self.stream = torch.cuda.current_stream(dev)

    def step(self, xin=None, o=None, s=None):
        from mixture_experts_ffn_09_b200 import moe
        w = self.w
        xin = self.x if xin is None else xin
        o = self.out if o is None else o
        s = self.stream if s is None else s
        if self.ext:
            moe.ffn_forward_ex(xin, self.router, self.gu, self.dn, w.E, w.K, w.norm_topk_prob,
                               self.act, o, self.sel, self.wts, self.rb, self.b1, self.b2, None,
                               self.ws, s, **self.ext)
        else:
            moe.ffn_forward(xin, self.router, self.gu, self.dn, w.E, w.K, w.norm_topk_prob,
                            self.act, o, self.sel, self.wts, self.rb, self.b1, self.b2, None,
                            self.ws, s)

    def expert_load(self):
        import numpy as np
        return np.bincount(self.sel.cpu().numpy().ravel(), minlength=self.w.E)


def time_steps(layer, steps, wd, world, local, what):
    """Device time of `steps` forwards between CUDA events on the launching
    stream, bracketed by a barrier and a synchronize; clocks sampled through
    NVML meanwhile.  Returns (ms of this rank, launches, clocks)."""
    import torch
    from mixture_experts_ffn_09_b200 import moe
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    wd.sync(f"before {what}")
    clocks = ClockSampler(local, pci_bus_id=cuda_pci_bus_id(local))
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    n_launch0 = moe.kernel_launches()
    t0.record(layer.stream)
    wd.run(steps, layer.step, what)
    t1.record(layer.stream)
    launches = moe.kernel_launches() - n_launch0
    wd.sync(what)
    clk = clocks.stop()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    return t0.elapsed_time(t1), launches, clk


def time_graph_steps(layer, steps, wd, world, what):
    """Device time of `steps` replays of one forward captured in a CUDA graph
    (the same C-ABI call, recorded once after the warm-up), back to back on
    the launching stream: the forward without the host's per-call work
    (argument checks in the binding, the library's host side, the launch).
    Returns ms of this rank over all replays."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    cap = torch.cuda.Stream(layer.dev)
    cap.wait_stream(layer.stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        main = layer.stream
        layer.stream = cap
        try:
            with torch.cuda.graph(g, stream=cap):
                layer.step()
        finally:
            layer.stream = main
    layer.stream.wait_stream(cap)
    for _ in range(3):
        g.replay()
    wd.sync(f"before {what}")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(layer.stream)
    for _ in range(steps):
        g.replay()
    t1.record(layer.stream)
    wd.sync(what)
    ms = t0.elapsed_time(t1)
    del g
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    return ms


def stage_pass(layer, n, wd, local, what):
    """Per-stage CUDA-event times of n forwards (events between the kernels
    on the launching stream, so not the headline number), with the clocks
    sampled through NVML during the pass.  Returns (ms per call by stage,
    clocks)."""
    from mixture_experts_ffn_09_b200 import moe
    clocks = ClockSampler(local, pci_bus_id=cuda_pci_bus_id(local))
    clocks.start()
    moe.profile_enable(True)
    wd.run(n, layer.step, what)
    wd.sync(what)
    stage_ms, calls = moe.profile_read()
    moe.profile_enable(False)
    clk = clocks.stop()
    return {k: v / max(calls, 1) for k, v in stage_ms.items()}, clk


def uses_pair_gemm(w, gemm: str) -> bool:
    return w.dtype == "bf16" and (gemm == "2sm" or (gemm == "auto" and w.T * w.K >= 512 * w.E))


FP32_LANES_PER_SM = 128             # fp32 FMA units per SM (4 sub-partitions x 32)


def alu_roofline(w, per_call, stage_clk):
    """Float32 layers run on CUDA cores: the dominant kernel (the one-kernel
    small layer, else the fp32 gate_up GEMM) against the fp32 FMA rate,
    148 SMs x 128 lanes x 2 FLOP per clock at the maximum SM clock."""
    small = per_call.get("small_layer", 0.0) > 0
    ms = per_call["small_layer"] if small else per_call["gate_up"]
    fl = w.routed_flops() if small else gate_up_flops(w)
    mhz = stage_clk.get("sm_max_mhz") or 1965
    peak = SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    achieved = fl / (ms / 1e3) / 1e12
    return {"kernel": "small_layer_f32_kernel (the whole layer, one cluster)" if small
            else "gemm_simt_f32_kernel<silu_gated> (gate_up, fp32 FMA)",
            "bound": "alu", "achieved": round(achieved, 4), "peak": round(peak, 2),
            "unit": "TFLOP/s", "frac": round(achieved / peak, 5),
            "peak_source": f"derived: {SMS} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 FLOP x {mhz} MHz",
            "algorithmic_flops_per_launch": fl, "avg_launch_ms": round(ms, 4)}


def gate_up_roofline(w, per_call, touched, peaks, gemm, timed_s, stage_clk):
    """Roofline of the dominant kernel, the gate_up grouped GEMM, from its
    CUDA-event time: routed FLOPs against the bf16 tensor peak at large T,
    the bytes it must move against the HBM copy bandwidth at small T."""
    if w.dtype != "bf16":
        return alu_roofline(w, per_call, stage_clk)
    t_gu = per_call["gate_up"] / 1e3
    pair = uses_pair_gemm(w, gemm)
    if w.dtype != "bf16":
        kname = "gemm_simt_f32_kernel<silu_gated> (gate_up, fp32 FMA)"
    elif pair:
        kname = "grouped_gemm_pair_kernel<silu_gated> (gate_up, CTA pairs)"
    else:
        kname = "grouped_gemm_tc_kernel<silu_gated> (gate_up, one CTA per tile)"
    if w.T * w.K <= 512:
        achieved = gate_up_bytes(w, touched) / t_gu / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "peak_source": peaks["source"] + " hbm copy",
                "frac_of_nominal_8tbs": round(achieved / NOMINAL["hbm_gbs"], 4),
                "algorithmic_bytes_per_launch": gate_up_bytes(w, touched)}
    else:
        fl = gate_up_flops(w)
        achieved = fl / t_gu / 1e12
        sustained = timed_s >= SUSTAINED_AFTER_S
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        roof = {"kernel": kname, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": peaks["source"] + (
                    " bf16 sustained (the timed loop lasted %.1f s)" % timed_s if sustained else
                    " bf16 burst (the timed loop lasted %.2f s, too short to settle at the power cap)"
                    % timed_s),
                "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4),
                "frac_of_sustained_peak": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "frac_of_datasheet_2250": round(achieved / NOMINAL["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": fl}
        mhz = stage_clk.get("sm_mhz")
        if mhz:
            per_clk = fl / (t_gu * mhz * 1e6)
            roof["achieved_per_clock"] = {
                "flop_per_clk": round(per_clk, 1), "sm_mhz": mhz,
                "peak_flop_per_clk": SMS * PEAK_FLOP_PER_CLK_PER_SM,
                "frac": round(per_clk / (SMS * PEAK_FLOP_PER_CLK_PER_SM), 4),
                "how": "gate_up FLOP / (CUDA-event time x median SM clock of the per-stage pass); "
                       "peak 148 SMs x 8192 dense bf16 FLOP per clock"}
    roof["avg_launch_ms"] = round(per_call["gate_up"], 4)
    return roof


def measure_extra(w, args, dev, local, world, peaks):
    """One more workload in the same process: its own inputs, warm-up,
    timed forwards and per-stage pass.  The numbers every config is judged
    on, without the end-to-end and CPU legs of the headline."""
    from mixture_experts_ffn_09_b200 import moe, synth
    d = synth.make_inputs(w)
    layer = Layer(w, d, dev, args)
    wd = Watchdog(dev, layer.stream, args.watchdog)
    for i in range(max(args.warmup, 3)):
        layer.step()
        wd.sync(f"{w.name} warm-up step {i}")
    st = moe.device_status(layer.stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{w.name}: device status after warm-up: {moe.status_string(st)}")
    load = layer.expert_load()
    touched = int((load > 0).sum())
    steps = max(5, min(args.steps, args.extra_steps))
    local_ms, launches, clk = time_steps(layer, steps, wd, world, local, f"{w.name} timed region")
    ms_step, tok_s = throughput(local_ms, steps, w.T, world, dev)
    # replays: at least ~50 ms of them (thousands for the microsecond-scale layers)
    g_steps = int(min(5000, max(steps, 50.0 / max(ms_step, 1e-3))))
    g_ms, g_tok_s = throughput(time_graph_steps(layer, g_steps, wd, world, f"{w.name} graph replays"),
                               g_steps, w.T, world, dev)
    per_call, sclk = stage_pass(layer, max(5, min(steps, 50)), wd, local, f"{w.name} per-stage pass")
    rflops = routed_flops(w)
    abytes = algorithmic_bytes(w, touched)
    r = {"config": workload_config(w, world), "steps": steps, "ms_per_step": round(ms_step, 4),
         "tokens_per_s": round(tok_s, 1), "routed_tflops": round(world * rflops / (ms_step / 1e3) / 1e12, 3),
         "stages_ms": {k: round(v, 4) for k, v in per_call.items()}, "gpu_launches": launches,
         "experts_touched": touched, "clocks": clk,
         "graph": {"ms_per_step": round(g_ms, 4), "tokens_per_s": round(g_tok_s, 1), "replays": g_steps,
                   "how": "the same forward captured once in a CUDA graph and replayed back to back "
                          "(no per-call host work); ms_per_step above is the direct C-ABI call"}}
    if w.dtype == "bf16":
        r["roofline"] = gate_up_roofline(w, per_call, touched, peaks, args.gemm, local_ms / 1e3, sclk)
        if w.T * w.K <= 512:
            # weight streaming: the whole step against the HBM copy bandwidth
            r["step_hbm"] = {"algorithmic_bytes": abytes,
                             "achieved_gbs": round(abytes / (ms_step / 1e3) / 1e9, 1),
                             "frac_of_copy": round(abytes / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                             "peak_source": peaks["source"],
                             "frac_of_nominal_8tbs": round(abytes / (ms_step / 1e3) / 1e9 / NOMINAL["hbm_gbs"], 4)}
        else:
            r["step_tensor"] = {
                "frac_of_burst_peak": round(rflops / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
                "frac_of_datasheet_2250": round(rflops / (ms_step / 1e3) / 1e12 / NOMINAL["bf16_tflops"], 4)}
    else:
        r["roofline"] = alu_roofline(w, per_call, sclk)
        r["bound"] = "latency (one small launch; inputs fit in L2)"
    del layer
    return r


def run_ours(args, w):
    import numpy as np
    import torch
    from mixture_experts_ffn_09_b200 import build, moe, synth

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    build.build()
    moe.set_gemm_mode({"auto": moe.GEMM_AUTO, "1sm": moe.GEMM_1SM, "2sm": moe.GEMM_2SM}[args.gemm])
    moe.set_pdl(args.pdl)
    moe.set_fused_gather(args.fused_gather)
    if args.tail_swap is not None:
        moe.set_tail_swap(args.tail_swap)
    tail_swap = moe.set_tail_swap(0)
    moe.set_tail_swap(tail_swap)
    if args.debug_sync_ms > 0:
        moe.set_debug_sync(args.debug_sync_ms)
    dev = torch.device("cuda", local)
    d = synth.make_inputs(w)

    ext = dict(score=args.score, dynamic_threshold=args.dynamic_threshold,
               capacity_factor=args.capacity_factor, seq_len=args.seq_len)
    if args.selection_bias > 0:
        sb = np.random.default_rng(7).normal(0, args.selection_bias, w.E).astype(np.float32)
        ext["selection_bias"] = torch.from_numpy(sb).to(dev)
    kept = torch.empty(w.T, w.K, dtype=torch.uint8, device=dev)
    bal = torch.empty(4, dtype=torch.float32, device=dev)
    use_ext = (args.score != "softmax" or args.selection_bias > 0 or args.dynamic_threshold > 0
               or args.capacity_factor > 0 or args.balance)
    if use_ext:
        ext["slot_kept"] = kept
        if args.balance:
            ext["balance"] = bal
    layer = Layer(w, d, dev, args, ext if use_ext else None)
    x, out, stream, dt = layer.x, layer.out, layer.stream, layer.dt
    step = layer.step

    wd = Watchdog(dev, stream, args.watchdog)
    for i in range(max(args.warmup, 3)):
        step()
        wd.sync(f"warm-up step {i}")
    st = moe.device_status(stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {moe.status_string(st)}")
    load = layer.expert_load()
    touched = int((load > 0).sum())
    ext_stats = {}
    if use_ext:
        k = kept.cpu().numpy()
        ext_stats["slots_kept_frac"] = round(float(k.mean()), 4)
        if args.balance:
            ext_stats["balance"] = dict(zip(("switch", "gshard", "master", "gshard_probs"),
                                            [round(float(v), 6) for v in bal.cpu().numpy()]))

    # ---------------- timed region: K forwards, device events on the stream
    local_ms, timed_launches, clk = time_steps(layer, args.steps, wd, world, local, "timed region")
    ms_step, tokens_per_s = throughput(local_ms, args.steps, w.T, world, dev)

    # ---------------- per-stage times: a separate pass with CUDA events
    # around every kernel on the launching stream (the events sit between
    # the kernels, so this pass is not the headline number), clocks sampled
    per_call, stage_clk = stage_pass(layer, max(20, min(args.steps, 50)), wd, local,
                                     "per-stage pass")
    st = moe.device_status(stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status after timing: {moe.status_string(st)}")

    # ---------------- end to end: pinned host x in, out back, every step
    # A serving loop: step i's input is uploaded on one copy stream while
    # step i-1 computes, and step i's output is read back on another while
    # step i+1 computes (two device buffers each); every step still moves
    # its own input and output bytes inside the timed region.  When a step's
    # copies are tiny (under 64 KB each way) the overlap saves nothing and
    # its stream and event calls cost more host time than the layer, so the
    # copies and the forward run in order on the compute stream instead.
    xh = _readonly_view(d["x"]).reshape(w.T, w.D).pin_memory()
    oh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    od = [torch.empty_like(out) for _ in range(2)]
    cs = torch.cuda.Stream(dev)                 # compute
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("up", "fwd", "down")}
    n_e2e = [0]
    io_bytes = w.T * w.D * (2 if dt == moe.BF16 else 4)
    serial = io_bytes < (64 << 10)

    def e2e_step_serial():
        b = n_e2e[0] & 1
        n_e2e[0] += 1
        with torch.cuda.stream(cs):
            xd[b].copy_(xh, non_blocking=True)
            step(xd[b], od[b], cs)
            oh[b].copy_(od[b], non_blocking=True)

    def e2e_step():
        i = n_e2e[0]
        n_e2e[0] += 1
        b = i & 1
        if i >= 2:
            up_s.wait_event(ev["fwd"][b])           # xd[b] is free once step i-2 computed
        with torch.cuda.stream(up_s):
            xd[b].copy_(xh, non_blocking=True)
        ev["up"][b].record(up_s)
        cs.wait_event(ev["up"][b])
        if i >= 2:
            cs.wait_event(ev["down"][b])            # od[b] is free once step i-2 was read back
        step(xd[b], od[b], cs)
        ev["fwd"][b].record(cs)
        down_s.wait_event(ev["fwd"][b])
        with torch.cuda.stream(down_s):
            oh[b].copy_(od[b], non_blocking=True)
        ev["down"][b].record(down_s)

    def e2e_drain():
        if serial:
            return
        for b in range(2):
            cs.wait_event(ev["down"][b])

    one_step = e2e_step_serial if serial else e2e_step

    e_steps = max(2, min(args.steps, 200))
    wd_cs = Watchdog(dev, cs, args.watchdog)
    for _ in range(3):
        one_step()
    e2e_drain()
    wd_cs.sync("end-to-end warm-up")
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    wd_cs.run(e_steps, one_step, "end-to-end region")
    e2e_drain()
    e1.record(cs)
    wd_cs.sync("end-to-end region")
    e_ms, e_tokens_per_s = throughput(e0.elapsed_time(e1), e_steps, w.T, world, dev)
    # the pipelined loop computed the same outputs as the device-resident one
    if not torch.equal(od[(n_e2e[0] - 1) & 1], out):
        raise RuntimeError("end-to-end output differs from the device-resident forward")

    # ---------------- roofline of the dominant kernel (gate_up)
    peaks = load_peaks()
    dom = max(per_call, key=per_call.get)
    roof = gate_up_roofline(w, per_call, touched, peaks, args.gemm, local_ms / 1e3, stage_clk)
    roof["traffic"] = (stored_traffic(w.name, "gate_up_pair" if uses_pair_gemm(w, args.gemm)
                                      else "gate_up") if w.dtype == "bf16" else None)
    roof["stage_pass_clocks"] = stage_clk

    rflops = routed_flops(w)
    abytes = algorithmic_bytes(w, touched)
    result = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded, shapes of the published workloads; random-init weights)",
        "config": dict(workload_config(w, world), gemm=args.gemm, pdl=args.pdl, tail_swap=tail_swap,
                       fused_gather=args.fused_gather,
                       **({"routing": {"score": args.score, "selection_bias_std": args.selection_bias,
                                       "dynamic_threshold": args.dynamic_threshold,
                                       "capacity_factor": args.capacity_factor,
                                       "seq_len": args.seq_len, "balance": args.balance}}
                          if use_ext else {})),
        "routed_tflops": round(world * rflops / (ms_step / 1e3) / 1e12, 2),
        "peaks": dict(peaks),
        "frac_of_bf16_peak": {
            "burst": round(rflops / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
            "sustained": round(rflops / (ms_step / 1e3) / 1e12 / peaks["bf16_tflops_sustained"], 4),
            "datasheet_2250": round(rflops / (ms_step / 1e3) / 1e12 / NOMINAL["bf16_tflops"], 4),
            "peak_source": peaks["source"]},
        "hbm": {"algorithmic_gb_per_step": round(abytes / 1e9, 4),
                "achieved_gbs": round(abytes / (ms_step / 1e3) / 1e9, 1),
                "frac_of_copy": round(abytes / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                "peak_source": peaks["source"],
                "frac_of_nominal_8tbs": round(abytes / (ms_step / 1e3) / 1e9 / NOMINAL["hbm_gbs"], 4)},
        "stages_ms": {k: round(v, 4) for k, v in per_call.items()},
        "dominant_stage": dom,
        "expert_load": load.tolist(), "experts_touched": touched, **ext_stats,
        "roofline": roof,
        "e2e": {"value": round(e_tokens_per_s, 1), "unit": UNIT,
                "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
                "ms_per_step": round(e_ms, 4),
                "how": ("per step, in order on the compute stream: pinned host x -> device, "
                        "moe_ffn_forward, out -> pinned host (copies under 64 KB: nothing to "
                        "overlap)" if serial else
                        "per step: pinned host x -> device on an upload stream, moe_ffn_forward on "
                        "a compute stream, out -> pinned host on a download stream; copies of "
                        "neighbouring steps overlap the forward (two device buffers each)")},
        "gpu_launches": timed_launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, secs = oracle_rate(w, d, args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(rate, 4), "unit": UNIT, "cores": cpu_cores(),
                                  "kind": "oracle",
                                  "sample": f"{n} tokens of the workload (from its start; the whole "
                                            f"batch repeated when it is quick), dense over all "
                                            f"{w.E} experts in float64 ({secs:.1f} s)"}
        if w.dtype == "f32":            # the small layers: one core as well
            r1, n1, s1 = oracle_rate_single_core(w, d, min(args.cpu_seconds, 10.0))
            result["cpu_baseline"]["single_core"] = {
                "value": round(r1, 4), "unit": UNIT, "cores": 1,
                "sample": f"{n1} tokens, BLAS held to one thread ({s1:.1f} s)"}

    # ---------------- every other config, same process, after the headline
    extra = [] if args.no_workloads else [synth.WORKLOADS[n] for n in EXTRA_WORKLOADS
                                          if n != w.name]
    if extra:
        del layer, xd, od, xh, oh
        torch.cuda.empty_cache()
        result["workloads"] = {}
        for ew in extra:
            result["workloads"][ew.name] = measure_extra(ew, args, dev, local, world, peaks)
            torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------- reference arm
def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    from mixture_experts_ffn_09_b200 import synth
    d = synth.make_inputs(w)
    # one step = the oracle on a bounded token sample; size it so that the
    # whole run stays within a few minutes
    total = args.steps + args.warmup
    rate0, n0, t0 = oracle_rate(w, d, budget_s=1.0, first_n=2)
    per_step_s = max(0.5, min(20.0, 150.0 / max(total, 1)))
    n = int(max(1, min(w.T, rate0 * per_step_s)))
    import numpy as np
    from oracle import moe_oracle as O
    x = synth.as_float32(d["x"]).reshape(-1, w.D)
    gu = synth.as_float32(d["gate_up_proj"]).astype(np.float64)
    dn = synth.as_float32(d["down_proj"]).astype(np.float64)
    rt = synth.as_float32(d["router"]).astype(np.float64)

    def step(i):
        lo = (i * n) % max(w.T - n + 1, 1)
        O.moe_ffn_forward(x[lo:lo + n], rt, gu, dn, w.K, w.norm_topk_prob, w.act, d["router_bias"],
                          d["b1"], d["b2"])

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    for i in range(args.steps):
        step(i)
    secs = time.perf_counter() - t
    rate = args.steps * n / secs
    cores = cpu_cores()
    sample = (f"{n} tokens per step (of {w.T}), dense over all {w.E} experts in float64, "
              f"{args.steps} steps in {secs:.1f} s")
    single = {}
    if w.dtype == "f32":                # the small layers: one core as well
        r1, n1, s1 = oracle_rate_single_core(w, d, 5.0)
        single = {"single_core": {"value": round(r1, 4), "unit": UNIT, "cores": 1,
                                  "sample": f"{n1} tokens, BLAS held to one thread ({s1:.1f} s)"}}
    print(json.dumps({
        "metric": METRIC, "value": round(rate, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / max(args.steps, 1) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, shapes of the published workloads; random-init weights)",
        "config": workload_config(w, 1), "impl": "reference",
        "cpu_baseline": dict({"value": round(rate, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                              "sample": sample}, **single),
        "e2e": {"value": round(rate, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    from mixture_experts_ffn_09_b200 import synth
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=synth.MIXTRAL.name, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample (cpu_baseline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only the selected workload (skip the other configs)")
    ap.add_argument("--extra-steps", type=int, default=100,
                    help="timed forwards of each other config (at most --steps)")
    ap.add_argument("--gemm", choices=["auto", "1sm", "2sm"], default="auto",
                    help="bf16 grouped GEMM: automatic, one CTA per tile, or CTA pairs")
    ap.add_argument("--score", choices=["softmax", "sigmoid"], default="softmax")
    ap.add_argument("--selection-bias", type=float, default=0.0,
                    help="std of a seeded per-expert selection-only bias (0: none)")
    ap.add_argument("--dynamic-threshold", type=float, default=0.0)
    ap.add_argument("--capacity-factor", type=float, default=0.0)
    ap.add_argument("--seq-len", type=int, default=0)
    ap.add_argument("--balance", action="store_true", help="also compute the balancing statistics")
    ap.add_argument("--tail-swap", type=int, default=None,
                    help="rows up to which an expert's last CTA-pair tile runs with swapped "
                         "operands (0..255, 0 = off; default: the library's)")
    ap.add_argument("--fused-gather", choices=["auto", "on", "off"], default="auto",
                    help="bf16 gate_up fetches token rows from x by index (moe_set_fused_gather; "
                         "default: the library's automatic choice)")
    ap.add_argument("--pdl", action="store_true",
                    help="launch the kernels with programmatic dependent launch (off by default)")
    ap.add_argument("--watchdog", type=float, default=120.0,
                    help="seconds any wait for the device may take before the run is ended")
    ap.add_argument("--debug-sync-ms", type=int, default=0,
                    help="wait (bounded) after every kernel and name the one that does not finish; "
                         "timings are then not meaningful")
    ap.add_argument("--deadline", type=float, default=900.0,
                    help="seconds after which the whole run dumps every thread's stack and exits")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    # last bound on the run: whatever blocks (a device wait, a driver call),
    # the process reports where and ends instead of holding the GPU
    import faulthandler
    faulthandler.dump_traceback_later(args.deadline, exit=True)
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return
    try:
        run_ours(args, w)
    except Exception as e:
        # a kernel may still be running: leave without the normal teardown,
        # whose device frees would wait for it
        import traceback
        traceback.print_exc()
        print(json.dumps({"error": f"{type(e).__name__}: {e}"}), flush=True)
        sys.stdout.flush()
        sys.stderr.flush()
        os._exit(3)


if __name__ == "__main__":
    main()
