"""Benchmark of the W4A4 dual-branch linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--report]
                    [--workload full|full_up|full_down|mid_up|mid_down|ffn0|ffn2|tiny|sweep
                                |ffn|ffn_mid]

One step is one pass of the whole path over one batch of synthetic input,
for every layer of the workload: calibration absmax of X and of W, the
finalisation (s, score, top-k), the weight pack, the activation prep and the
dual-branch GEMM -- all through the C-ABI of libw4a4.  The default workload
is T = 57600 tokens (16 x 45 x 80 latent positions) on the FFN up-projection
shape (5120 -> 13824, k = 32) and on the down-projection shape (13824 ->
5120, k = 64), each layer with its own synthetic input.  The ffn workloads
instead time the online FFN forward with the fused epilogue.

``value`` is whole-step effective TFLOPS, 2 T d_in d_out summed over the
layers divided by the step time (outlier columns counted at the 4-bit
rate).  Per-kernel numbers come from CUDA events recorded on the launching
stream around each launch inside the timed region.  The full workload's
inputs are larger than L2 (X is 590 MB / 1.59 GB), so nothing is flushed;
where a step's inputs are under twice the L2 size a 256 MB buffer is written
between steps, outside each step's own events.  ``e2e`` times the online
layer through the library's host-buffer call (w4a4_linear_host: upload of X,
prep, GEMM, download of Y in one call per layer), with the copies inside the
timed region; the offline half's device time is reported beside it.  The
default line also carries ``context_ffn``: the FFN pair (up, GELU, down) at
T = 57600, fused against unfused, timed after everything else
(``--no-ffn-context`` skips it).

``--gpus N`` runs N ranks, one per GPU: launched without a launcher around it,
bench.py starts them itself through torch's launcher (rendezvous on
127.0.0.1); under torchrun it runs as the rank it is given.  Each rank runs
the same per-GPU workload on its own token shard (weak scaling, no collective
on the data path); the step time is the max over ranks, ``value`` counts the
work of all ranks.

``--report`` prints one JSON line per configuration (tiny, ffn.0, ffn.2, the
two full layers, every sweep point) with the GEMM's TFLOPS and fraction of
peak, the prep kernel's GB/s, the SNR of Y against the unquantised float64
X W^T, a cuBLAS bf16 GEMM of the same shape and the oracle on a sample.

``--impl reference`` times the CPU oracle (the numpy reference the tests
check the GPU against) on a bounded row sample of the same workload, on
rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dual-branch W4A4 GEMM TFLOPS & % of FP4 peak; prep kernel HBM GB/s"
LAYOUT_NAMES = {0: "32x1", 1: "32x32", 2: "128x1"}
FP4_NOMINAL_TFLOPS = 9000.0        # B200 dense FP4, datasheet
FP4_PER_BF16 = 4.0                 # nominal dense FP4 : BF16 ratio (9 / 2.25 PFLOP/s)
HBM_NOMINAL_GBS = 8000.0


# ---------------------------------------------------------------------------
# distributed plumbing (host only; covered by gloo tests on CPU)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(backend: str, world: int, rank: int, timeout_s: float = 120.0):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, world_size=world, rank=rank,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return world > 1


def dist_barrier(active: bool, device=None):
    import torch.distributed as dist
    if active:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def dist_max(value: float, active: bool, device) -> float:
    """Max of a float over ranks (every rank calls it)."""
    if not active:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, world: int, step_s_max: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return per_rank_units * world / step_s_max


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class NvmlClockSampler:
    """SM clock, power and clock-event reasons read through NVML every 5 ms in a
    background thread (the same counters nvidia-smi prints; reading them
    changes nothing).  Only samples inside the timed window are summarised."""
    REASONS = (("hw_slowdown", 0x8), ("hw_power_brake_slowdown", 0x80),
               ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, handle, nvml):
        self.h = handle
        self.nvml = nvml
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = None
        self.window = (None, None)
        self.max_mhz = None

    @staticmethod
    def open(local_index: int):
        """An NVML sampler for CUDA device `local_index`, or None."""
        try:
            import pynvml as nvml
            import torch
            nvml.nvmlInit()
            prop = torch.cuda.get_device_properties(local_index)
            bus = getattr(prop, "pci_bus_id", None)
            if bus is not None:
                busid = "%08X:%02X:%02X.0" % (getattr(prop, "pci_domain_id", 0), bus,
                                              getattr(prop, "pci_device_id", 0))
                h = nvml.nvmlDeviceGetHandleByPciBusId(busid)
            else:
                h = nvml.nvmlDeviceGetHandleByIndex(local_index)
            nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM)
            return NvmlClockSampler(h, nvml)
        except Exception:
            return None

    def start(self):
        try:
            self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
        except Exception:
            self.max_mhz = None
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        n = self.nvml
        while not self.stop_evt.is_set():
            try:
                self.samples.append((time.time(), float(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)),
                                     n.nvmlDeviceGetPowerUsage(self.h) / 1000.0,
                                     int(n.nvmlDeviceGetCurrentClocksEventReasons(self.h))))
            except Exception:
                pass
            time.sleep(0.005)

    def mark_start(self):
        self.window = (time.time(), None)

    def mark_end(self):
        self.window = (self.window[0], time.time())

    def stop(self):
        self.stop_evt.set()
        if self.thread:
            self.thread.join(timeout=2)
        t0, t1 = self.window
        inside = [x for x in self.samples if t0 is not None and t1 is not None and t0 <= x[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": ["no samples in the timed window"], "samples_total": len(self.samples),
                    "source": "nvml, 5 ms"}
        reasons = sorted({name for _, _, _, r in inside for name, bit in self.REASONS if r & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside),
                "sm_min_mhz": min(x[1] for x in inside),
                "sm_max_mhz": self.max_mhz if self.max_mhz else max(x[1] for x in inside),
                "power_w_max": max(x[2] for x in inside), "samples": len(inside),
                "reasons": reasons, "source": "nvml, 5 ms"}


def clock_sampler(local_index: int):
    """NVML sampling where it works, nvidia-smi otherwise."""
    s = NvmlClockSampler.open(local_index)
    return s if s is not None else ClockSampler(local_index)


class ClockSampler:
    """nvidia-smi samples every 20 ms; only samples whose timestamp falls inside
    the timed window are summarised."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.window = (None, None)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark_start(self):
        self.window = (time.time(), None)

    def mark_end(self):
        self.window = (self.window[0], time.time())

    @staticmethod
    def _ts(text):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        t0, t1 = self.window
        sm, smax, power, reasons, total = [], [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            total += 1
            ts = self._ts(p[0])
            if ts is not None and t0 is not None and t1 is not None and not (t0 <= ts <= t1):
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
                power.append(float(p[3]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples in the timed window"],
                    "samples_total": total}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of
# gemm_dual_pair_kernel, from one ncu capture each of the mid-size layers
# (T = 16384: the up layer 5120 -> 13824 and the down layer 13824 -> 5120;
# counter captures are kept to mid-size workloads).  Every DRAM stream of the
# GEMM grows in proportion to T (A, its scales and X_O are read once per
# 384- or 256-column tile sweep, B once per raster group of M tiles, Y
# written once), so a full-workload launch is the mean of the two captures
# times 57600 / 16384.  Valid only for the GEMM sources with this SHA-256
# (gemm.cu then w4a4_device.cuh); reported as null for any other source or
# workload.
GEMM_TRAFFIC = {
    "sha256": "d128d573ac3fd7cf4f693eb9eef4ff76026aa6009a48c6bcb2f5878b95f3af41",
    "workload": "full",
    "mid_bytes": {"up": 169650176 + 408704512, "down": 320878080 + 149832960},
    "scale": 57600 / 16384,
}


def gemm_traffic(workload: str):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "w4a4_mxfp4_outlier_b200", "csrc")
    for f in ("gemm.cu", "w4a4_device.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != GEMM_TRAFFIC["sha256"] or workload != GEMM_TRAFFIC["workload"]:
        return None
    mid = GEMM_TRAFFIC["mid_bytes"]
    return int((mid["up"] + mid["down"]) / 2 * GEMM_TRAFFIC["scale"])


def peak_keys(timed_seconds: float):
    """(peak used, the other one): the burst bf16 figure for a timed region
    shorter than a second of back-to-back work (the measured burst figure is
    the best of ten sub-millisecond GEMMs), the sustained one (measured over a
    4 s loop under the power cap) for longer regions."""
    if timed_seconds >= 1.0:
        return "bf16_tflops_sustained", "bf16_tflops"
    return "bf16_tflops", "bf16_tflops_sustained"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def layer_bytes_prep(L, d) -> float:
    """Algorithmic bytes of the prep kernel: X read + codes, scales and X_O written."""
    return L.T * (2.0 * L.d_in + d.kj_pad / 2 + d.nblk + 2.0 * d.k_pad)


class LayerRun:
    """Device buffers and the C-ABI call sequence of one layer."""

    def __init__(self, L, device, w4, synth):
        import torch
        self.L = L
        self.w4 = w4
        self.X, self.W = synth.gen_layer(L, device)
        self.pw = w4.alloc_packed(L.d_in, L.d_out, L.k, L.layout, device)
        self.act = w4.alloc_act(L.T, self.pw)
        self.Y = torch.empty((L.T, L.d_out), dtype=torch.bfloat16, device=device)
        self.d = self.pw.dims
        self.launches = 0

    def offline(self, ev=None):
        """Calibration (absmax of X and W), finalisation and packing."""
        w4, L, pw = self.w4, self.L, self.pw
        if ev is not None:
            ev[0].record()
        w4.calib_observe_layer(self.X, self.W, pw.act_scale, pw.w_scale, reset=True)
        if ev is not None:
            ev[1].record()
        w4.calib_finalize(pw.act_scale, pw.w_scale, L.alpha, L.k, pw.s, pw.inv_s, pw.score,
                          pw.O if L.k else None, pw.jmap if L.k < L.d_in else None)
        w4.pack_weight(self.W, pw)
        # colabsmax (X and W), finalize x2, pack: one prep launch (32x1) or tile + bf16 kernels (32x32)
        pack = 1 if L.layout in (0, 2) else (1 if self.d.kj else 0) + (1 if L.k else 0)
        return 3 + pack

    def online(self, ev=None):
        w4 = self.w4
        if ev is not None:
            ev[0].record()
        w4.prep_act(self.X, self.pw, self.act)
        if ev is not None:
            ev[1].record()
        w4.gemm_dual(self.act, self.L.T, self.pw, self.Y)
        if ev is not None:
            ev[2].record()
        return 2


def check_device(local: int):
    """One rank per GPU: a rank whose local index has no GPU stops here (two
    ranks on one GPU are not run)."""
    import torch
    n = torch.cuda.device_count()
    if local >= n:
        raise SystemExit(f"bench.py: rank with LOCAL_RANK={local} has no GPU "
                         f"({n} visible); run at most {n} ranks")


def cublas_bf16_context(runs, reps=5):
    """cuBLAS bf16 GEMM of the same shapes (Y = X W^T through torch.mm), timed
    after the timed region as context: the unquantised product this path
    replaces.  Returns the mean milliseconds per layer."""
    import torch
    out = []
    for r in runs:
        Yc = torch.empty_like(r.Y)
        for _ in range(2):
            torch.mm(r.X, r.W.t(), out=Yc)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            torch.mm(r.X, r.W.t(), out=Yc)
        b.record()
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b) / reps)
        del Yc
    return out


def run_gpu(args):
    import torch

    import synth
    import w4a4_mxfp4_outlier_b200 as w4

    world, rank, local = dist_env()
    check_device(local)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    active = dist_init("nccl", world, rank)
    layers = [L.with_(seed=L.seed + 1000 * rank) for L in synth.WORKLOADS[args.workload]]
    runs = [LayerRun(L, device, w4, synth) for L in layers]
    torch.cuda.synchronize()

    def step(evs=None):
        n = 0
        for i, r in enumerate(runs):
            n += r.offline(None if evs is None else evs[i]["off"])
            n += r.online(None if evs is None else evs[i]["on"])
        return n

    for _ in range(args.warmup):
        step()
    st, bits = w4.last_error()
    if st != w4.OK:
        raise RuntimeError(f"device error word {bits:#x} during warm-up")

    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [[{"off": [mk(), mk()], "on": [mk(), mk(), mk()]} for _ in runs] for _ in range(args.steps)]
    t0, t1 = mk(), mk()
    flush = l2_flush_buffer(min(layer_input_bytes(L) for L in layers), device)
    s_evs = [(mk(), mk()) for _ in range(args.steps)]
    clocks = clock_sampler(local)
    torch.cuda.synchronize()
    dist_barrier(active, device)
    clocks.start()
    time.sleep(0.2)
    clocks.mark_start()
    t0.record()
    launches = 0
    for k in range(args.steps):
        if flush is not None:
            flush.zero_()                       # between steps, outside the step's events
        s_evs[k][0].record()
        launches += step(evs[k])
        s_evs[k][1].record()
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    clock_info = clocks.stop()
    dist_barrier(active, device)
    st, bits = w4.last_error()
    if st != w4.OK:
        raise RuntimeError(f"device error word {bits:#x} in the timed region")

    step_ms = sum(a.elapsed_time(b) for a, b in s_evs) / args.steps
    step_ms_max = dist_max(step_ms, active, device)
    flops = sum(L.flops for L in layers)
    value = aggregate(flops, world, step_ms_max * 1e-3) / 1e12

    gemm_ms = [sum(e[i]["on"][1].elapsed_time(e[i]["on"][2]) for e in evs) / args.steps
               for i in range(len(runs))]
    prep_ms = [sum(e[i]["on"][0].elapsed_time(e[i]["on"][1]) for e in evs) / args.steps
               for i in range(len(runs))]
    calib_ms = [sum(e[i]["off"][0].elapsed_time(e[i]["off"][1]) for e in evs) / args.steps
                for i in range(len(runs))]
    offline_ms = [sum(e[i]["off"][0].elapsed_time(e[i]["on"][0]) for e in evs) / args.steps
                  for i in range(len(runs))]
    gemm_tflops = flops / (sum(gemm_ms) * 1e-3) / 1e12
    prep_bytes = sum(layer_bytes_prep(r.L, r.d) for r in runs)
    prep_gbs = prep_bytes / (sum(prep_ms) * 1e-3) / 1e9
    calib_bytes = sum(2.0 * (r.L.T * r.L.d_in + r.L.d_out * r.L.d_in) for r in runs)
    calib_gbs = calib_bytes / (sum(calib_ms) * 1e-3) / 1e9
    online_tflops = flops / ((sum(gemm_ms) + sum(prep_ms)) * 1e-3) / 1e12

    peaks, src = measured_peaks()
    key, other_key = peak_keys(step_ms * args.steps * 1e-3)
    fp4_peak = peaks[key] * FP4_PER_BF16
    other = peaks[other_key] * FP4_PER_BF16
    roof = {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
            "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
            "traffic": gemm_traffic(args.workload),
            "traffic_unit": "bytes per launch (ncu dram read + write on T=16384, scaled to T=57600)",
            "kernel": "gemm_dual_pair_kernel",
            "peak_source": f"{src}: {key} x {FP4_PER_BF16:g} (nominal FP4:BF16 ratio), of measured",
            "frac_of_other_peak": round(gemm_tflops / other, 4),
            "frac_of_nominal_fp4_9pf": round(gemm_tflops / FP4_NOMINAL_TFLOPS, 4)}

    cublas_ms = cublas_bf16_context(runs)
    e2e = run_e2e(args, runs, w4, device, active) if not args.no_e2e else None
    if e2e is not None:
        e2e["offline_ms"] = [round(x, 4) for x in offline_ms]
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(layers, runs, rows=256, outs=1024)
    ffn_ctx = None
    if rank == 0 and args.workload == "full" and not args.no_ffn_context:
        try:                                      # context only: it never costs the headline line
            ffn_ctx = ffn_context(device)
        except Exception as e:                    # noqa: BLE001
            ffn_ctx = {"error": f"{type(e).__name__}: {e}"[:300]}

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1/e8m0 x e2m1/e8m0 + bf16 x bf16, f32 accumulate",
            "data": "synthetic (seeded heavy-tailed X, clipped-normal W; see synth/)",
            "config": layer_workload_config(args.workload, layers, world, flush is not None),
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clock_info,
            "kernels": {
                "gemm_ms": [round(x, 4) for x in gemm_ms],
                "gemm_tflops": round(gemm_tflops, 1),
                "prep_ms": [round(x, 4) for x in prep_ms],
                "prep_gbs": round(prep_gbs, 1),
                "prep_frac_hbm_measured": round(prep_gbs / peaks["hbm_gbs"], 4),
                "prep_frac_hbm_nominal_8tbs": round(prep_gbs / HBM_NOMINAL_GBS, 4),
                "calib_absmax_ms": [round(x, 4) for x in calib_ms],
                "calib_absmax_gbs": round(calib_bytes / (sum(calib_ms) * 1e-3) / 1e9, 1),
                "online_tflops": round(online_tflops, 1),
            },
            "context_cublas_bf16": {
                "gemm_ms": [round(x, 4) for x in cublas_ms],
                "tflops": round(flops / (sum(cublas_ms) * 1e-3) / 1e12, 1),
                "dual_gemm_speedup": round(sum(cublas_ms) / sum(gemm_ms), 3),
                "note": "torch.mm bf16 of the same X and W, timed after the timed region "
                        "(5 reps, L2 not flushed); not part of the step"},
        }
        if ffn_ctx is not None:
            out["context_ffn"] = ffn_ctx
        print(json.dumps(out), flush=True)
    if active:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, runs, w4, device, active):
    """The online layer end to end through the library's host-buffer call,
    w4a4_linear_host: each call copies X from pinned host memory to the
    device, runs the activation prep and the dual-branch GEMM, and copies Y
    back to pinned host memory, all enqueued by the library on the stream it
    is given.  A step is one such call per layer of the workload.  Two buffer
    sets per layer on two streams alternate between consecutive steps, so one
    step's uploads overlap the previous step's compute and downloads (PCIe is
    full duplex).  The offline half (calibration and pack, once per layer in
    deployment) ran before the timed region; its device time is in the main
    line's kernels (calib_absmax_ms) and in offline_ms below."""
    import torch
    sets = []
    for r in runs:
        xh = r.X.cpu().pin_memory()
        per = []
        for _ in range(2):
            per.append({"xd": torch.empty_like(r.X), "yd": torch.empty_like(r.Y),
                        "yh": torch.empty(r.Y.shape, dtype=r.Y.dtype).pin_memory(),
                        "ws": torch.empty(w4.workspace_size(r.L.T, r.L.d_in, r.L.d_out, r.L.k),
                                          dtype=torch.uint8, device=device),
                        "stream": torch.cuda.Stream(device)})
        sets.append((xh, per))
    h2d = sum(r.L.T * r.L.d_in * 2 for r in runs)
    d2h = sum(r.L.T * r.L.d_out * 2 for r in runs)
    steps = max(3, min(args.steps, 8))
    calls = [0]

    def step(k):
        for r, (xh, per) in zip(runs, sets):
            b = per[k % 2]
            w4.linear_host(xh, r.pw, b["xd"], b["ws"], b["yd"], b["yh"], stream=b["stream"])
            calls[0] += 1

    def join(s):
        for _, per in sets:
            for b in per:
                s.wait_stream(b["stream"])

    main_s = torch.cuda.current_stream(device)
    step(0)
    step(1)
    torch.cuda.synchronize()
    # the step's Y arrived on the host, bit for bit what the device path gives
    for r, (_, per) in zip(runs, sets):
        if not torch.equal(per[1]["yh"], r.Y.cpu()):
            raise RuntimeError(f"{r.L.name}: linear_host output differs from the device path")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    dist_barrier(active, device)
    t0.record(main_s)
    for _, per in sets:
        for b in per:
            b["stream"].wait_stream(main_s)
    calls[0] = 0
    for k in range(steps):
        step(k)
    join(main_s)
    t1.record(main_s)
    torch.cuda.synchronize()
    ms = dist_max(t0.elapsed_time(t1) / steps, active, device)
    world = dist_env()[0]
    flops = sum(r.L.flops for r in runs)
    return {"value": round(aggregate(flops, world, ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
            "ms_per_step": round(ms, 3), "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "h2d_gbs": round(h2d / (ms * 1e-3) / 1e9, 1),
            "d2h_gbs": round(d2h / (ms * 1e-3) / 1e9, 1),
            "path": "w4a4_linear_host per layer and step (H2D of X, prep, dual GEMM, D2H of Y, "
                    "all enqueued by the library), two buffer sets per layer on alternating "
                    "streams",
            "calls_per_step": calls[0] // steps,
            "offline": "calibration and pack once per layer before the timed region "
                       "(device time reported as offline_ms)"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
def _threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(layers, rows_per_layer=64, out_per_layer=256, X_rows=None, W_rows=None):
    """Run the oracle's whole path on a row sample of each layer.

    Calibration sees the sampled rows, the pack covers `out_per_layer` output
    channels, prep and the product the sampled tokens.  Returns (effective
    FLOPs of the sample, seconds)."""
    import numpy as np

    from oracle import w4a4_oracle as orc
    flops, secs = 0.0, 0.0
    for i, L in enumerate(layers):
        X = X_rows[i]
        W = W_rows[i]
        t = time.perf_counter()
        c = orc.calibrate(X, W, L.alpha, L.k)
        pw = orc.pack_weight(W, c["s"], c["O"], c["J"], L.layout)
        pa = orc.prep_activation(X, c["inv_s"], c["O"], c["J"])
        Y = orc.dual_branch_product(pa["aq"], pa["sfa"], pa["xo"], pw["wq"], pw["sfb"], pw["w_hp"])
        secs += time.perf_counter() - t
        flops += 2.0 * X.shape[0] * L.d_in * W.shape[0]
        assert np.isfinite(Y).all()
    return flops, secs


def _host_samples(layers, runs=None, rows=64, outs=256):
    import torch

    import synth
    Xs, Ws = [], []
    for i, L in enumerate(layers):
        if runs is not None:
            X, W = runs[i].X, runs[i].W
        else:
            X = synth.gen_x(L.x, min(L.T, 2048), L.d_in, L.seed)
            W = synth.gen_w(L.w, min(L.d_out, 2048), L.d_in, L.seed + 1)
        idx = synth.sample_rows(X.shape[0], rows)
        Xs.append(X[idx.to(X.device)].float().cpu().numpy())
        Ws.append(W[:outs].float().cpu().numpy())
    _ = torch
    return Xs, Ws


def cpu_baseline(layers, runs=None, rows=64, outs=256):
    Xs, Ws = _host_samples(layers, runs, rows, outs)
    flops, secs = oracle_sample(layers, rows, outs, Xs, Ws)
    return {"value": round(flops / secs / 1e12, 8), "unit": "TFLOPS", "cores": _threads_used(),
            "kind": "oracle",
            "sample": f"{rows} token rows x {outs} output channels per layer, whole path "
                      f"(calibrate, pack, prep, product) in numpy; {secs:.1f} s"}


L2_BYTES = 126e6     # B200 L2


def layer_input_bytes(L) -> float:
    """A layer step's inputs: X and W, bf16."""
    return 2.0 * (L.T * L.d_in + L.d_out * L.d_in)


def l2_flush_buffer(input_bytes: float, device):
    """A 256 MB buffer to overwrite L2 between timed steps when a step's inputs
    are under twice the L2 size, else None (the inputs flush it themselves)."""
    if input_bytes >= 2 * L2_BYTES:
        return None
    import torch
    return torch.empty(256 << 20, dtype=torch.uint8, device=device)


def l2_note(flushed: bool) -> str:
    return ("L2 flushed between steps: 256 MB written outside the steps' events" if flushed
            else "inputs larger than L2 (no flush)")


def layer_workload_config(workload, layers, world, flushed=None):
    """The `config` of a layer workload's JSON line (both arms print the same)."""
    if flushed is None:
        flushed = min(layer_input_bytes(L) for L in layers) < 2 * L2_BYTES
    return {"workload": f"{workload}: " + ", ".join(
                f"{L.name} T={L.T} {L.d_in}->{L.d_out} k={L.k} alpha={L.alpha} "
                f"{LAYOUT_NAMES[L.layout]}" for L in layers),
            "tokens_per_gpu": layers[0].T, "parallelism": f"token shards x{world}",
            "l2": l2_note(flushed),
            "step": "calib absmax X,W + finalize + pack + prep + dual GEMM per layer"}


def ffn_input_bytes(Lu) -> float:
    """An FFN step's input: X, bf16 (the weights are packed before timing)."""
    return 2.0 * Lu.T * Lu.d_in


def ffn_workload_config(workload, Lu, Ld, world, flushed=None):
    """The `config` of an FFN workload's JSON line (both arms print the same)."""
    if flushed is None:
        flushed = ffn_input_bytes(Lu) < 2 * L2_BYTES
    return {"workload": f"{workload}: T={Lu.T} {Lu.d_in}->{Lu.d_out} k={Lu.k} alpha={Lu.alpha}, GELU, "
                        f"{Lu.d_out}->{Lu.d_in} k={Ld.k} alpha={Ld.alpha}, {LAYOUT_NAMES[Lu.layout]}",
            "tokens_per_gpu": Lu.T, "parallelism": f"token shards x{world}",
            "l2": l2_note(flushed),
            "step": "online FFN forward, fused: prep + up GEMM with GELU/prep epilogue "
                    "+ down GEMM (packed weights prepared before timing)"}


def report_layers():
    """The configurations of the report: tiny, ffn.0 and ffn.2 at T = 4096,
    the two layers of the full T = 57600 workload, every sweep point."""
    import synth
    return ([synth.TINY, synth.FFN0, synth.FFN2, synth.FULL_UP, synth.FULL_DOWN]
            + synth.sweep_layers())


def snr_db(Y, Y_exact) -> float:
    """10 log10(sum Y_exact^2 / sum (Y - Y_exact)^2)."""
    import numpy as np
    num = float(np.sum(Y_exact * Y_exact))
    den = float(np.sum((Y - Y_exact) ** 2))
    return 10.0 * np.log10(num / den) if den > 0 else float("inf")


def run_report(args):
    """One JSON line per configuration: the dual GEMM's TFLOPS and fraction of
    the FP4 peak, the prep kernel's GB/s and fraction of the HBM copy
    bandwidth, the SNR of Y against the unquantised float64 X W^T on sampled
    rows (reported, not a pass criterion), a cuBLAS bf16 GEMM of the same
    shape as context, and the CPU oracle on a row sample.  Single GPU."""
    import numpy as np
    import torch

    import synth
    import w4a4_mxfp4_outlier_b200 as w4
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("bench.py --report runs on one GPU")
    check_device(local)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    peaks, src = measured_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    mk = lambda: torch.cuda.Event(enable_timing=True)
    for L in report_layers():
        r = LayerRun(L, device, w4, synth)
        for _ in range(args.warmup):
            r.offline()
            r.online()
        flush = l2_flush_buffer(layer_input_bytes(L), device)
        evs = [[mk(), mk(), mk()] for _ in range(args.steps)]
        clocks = clock_sampler(local)
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.05)
        clocks.mark_start()
        for k in range(args.steps):
            r.offline()
            if flush is not None:
                flush.zero_()
            r.online(evs[k])
        torch.cuda.synchronize()
        clocks.mark_end()
        clock_info = clocks.stop()
        st, bits = w4.last_error()
        if st != w4.OK:
            raise RuntimeError(f"{L.name}: device error word {bits:#x}")
        gemm_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
        prep_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
        gemm_tflops = L.flops / (gemm_ms * 1e-3) / 1e12
        prep_gbs = layer_bytes_prep(L, r.d) / (prep_ms * 1e-3) / 1e9
        rows = synth.sample_rows(L.T, 256)
        ridx = rows.to(device)
        Xr = r.X[ridx].double().cpu().numpy()
        exact = Xr @ r.W.double().cpu().numpy().T
        snr = snr_db(r.Y[ridx].double().cpu().numpy(), exact)
        cub_ms = cublas_bf16_context([r])[0]
        Xs, Ws = _host_samples([L], [r], 64, 256)
        of, osec = oracle_sample([L], 64, 256, Xs, Ws)
        out = {"report": L.name,
               "config": f"T={L.T} {L.d_in}->{L.d_out} k={L.k} alpha={L.alpha} "
                         f"{LAYOUT_NAMES[L.layout]}",
               "steps": args.steps, "warmup": args.warmup, "l2": l2_note(flush is not None),
               "gemm_ms": round(gemm_ms, 4), "gemm_tflops": round(gemm_tflops, 1),
               "gemm_frac_fp4_peak": round(gemm_tflops / fp4_peak, 4),
               "gemm_frac_fp4_nominal_9pf": round(gemm_tflops / FP4_NOMINAL_TFLOPS, 4),
               "fp4_peak": f"{src} bf16_tflops x {FP4_PER_BF16:g} = {fp4_peak:.1f} TFLOP/s",
               "prep_ms": round(prep_ms, 4), "prep_gbs": round(prep_gbs, 1),
               "prep_frac_hbm_measured": round(prep_gbs / peaks["hbm_gbs"], 4),
               "prep_frac_hbm_nominal_8tbs": round(prep_gbs / HBM_NOMINAL_GBS, 4),
               "snr_db_vs_fp64_xw": round(snr, 2), "snr_rows": int(rows.numel()),
               "cublas_bf16_ms": round(cub_ms, 4),
               "cublas_bf16_tflops": round(L.flops / (cub_ms * 1e-3) / 1e12, 1),
               "clocks": clock_info,
               "oracle": {"seconds": round(osec, 2), "tflops": round(of / osec / 1e12, 8),
                          "cores": _threads_used(),
                          "sample": "64 token rows x 256 output channels, whole path in numpy"}}
        print(json.dumps(out), flush=True)
        del r, flush, Xr, exact
        torch.cuda.empty_cache()


def run_reference(args):
    import synth
    world, rank, _ = dist_env()
    if rank != 0:
        return
    # the FFN workloads: the same two layers, each sampled on its own input
    name = {"ffn": "full", "ffn_mid": "mid_up"}.get(args.workload, args.workload)
    layers = list(synth.WORKLOADS[name]) if name != "mid_up" else [synth.MID_UP, synth.MID_DOWN]
    Xs, Ws = _host_samples(layers, None, 64, 256)
    for _ in range(args.warmup):
        oracle_sample(layers, 64, 256, Xs, Ws)
    tot_f, tot_s = 0.0, 0.0
    for _ in range(args.steps):
        f, s = oracle_sample(layers, 64, 256, Xs, Ws)
        tot_f += f
        tot_s += s
    v = tot_f / tot_s / 1e12
    cores = _threads_used()
    sample = ("64 token rows x 256 output channels per layer of the workload, whole path "
              "(calibrate, pack, prep, product) in the numpy oracle")
    if args.workload in ("ffn", "ffn_mid"):
        sample += ("; the FFN's up and down layers each on its own synthetic input (the GELU "
                   "between them is not part of the sample)")
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 8), "unit": "TFLOPS",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(tot_s / args.steps * 1e3, 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64 (numpy oracle)",
           "data": "synthetic",
           "config": (ffn_workload_config(args.workload, layers[0], layers[1], world)
                      if args.workload in ("ffn", "ffn_mid")
                      else layer_workload_config(args.workload, layers, world)),
           "cpu_baseline": {"value": round(v, 8), "unit": "TFLOPS", "cores": cores,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(v, 8), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def ffn_setup(Lu, Ld, device, rank=0):
    """Inputs, calibration and packing of the FFN pair (up layer Lu, down
    layer Ld, the down layer fed by the up layer's output), and the two
    forwards: fused (prep, up GEMM whose epilogue writes the down layer's
    quantised activations, down GEMM; returns its launch count) and unfused
    (up linear to bf16 Y, GELU, down linear).  Returns (fused, unfused, Y of
    the fused forward, Y of the unfused one)."""
    import torch

    import synth
    import w4a4_mxfp4_outlier_b200 as w4
    from w4a4_mxfp4_outlier_b200 import ffn

    T, d_model, d_ff = Lu.T, Lu.d_in, Lu.d_out
    X, W_up = synth.gen_layer(Lu, device)
    W_down = synth.gen_w(Ld.w, Ld.d_out, Ld.d_in, seed=Ld.seed + 1 + 1000 * rank, device=device)
    f = ffn.calibrate_ffn(X, W_up, W_down, Lu.alpha, Lu.k, Ld.alpha, Ld.k, Lu.layout)
    act_up, act_down = w4.alloc_act(T, f.up), w4.alloc_act(T, f.down)
    Y = torch.empty((T, d_model), dtype=torch.bfloat16, device=device)
    ws_u = torch.empty(w4.workspace_size(T, d_model, d_ff, Lu.k), dtype=torch.uint8, device=device)
    ws_d = torch.empty(w4.workspace_size(T, d_ff, d_model, Ld.k), dtype=torch.uint8, device=device)
    Yu = torch.empty((T, d_ff), dtype=torch.bfloat16, device=device)
    H = torch.empty((T, d_ff), dtype=torch.bfloat16, device=device)
    Y2 = torch.empty_like(Y)

    def fused(ev=None):
        if ev: ev[0].record()
        w4.prep_act(X, f.up, act_up)
        if ev: ev[1].record()
        ffn.gemm_dual_act(act_up, T, f, act_down)
        if ev: ev[2].record()
        w4.gemm_dual(act_down, T, f.down, Y)
        if ev: ev[3].record()
        return 3

    def unfused():
        w4.linear(X, f.up_plain, ws_u, Yu)
        ffn.gelu_bf16(Yu, H)
        w4.linear(H, f.down, ws_d, Y2)

    return fused, unfused, Y, Y2


def ffn_context(device, steps=10, warmup=3):
    """The FFN pair at T=57600 (fused against unfused), timed after the
    headline line's own measurements as context: the measurement of
    `--workload ffn`, without its clock sampling and L2 logic (its inputs are
    larger than L2)."""
    import torch

    import synth
    import w4a4_mxfp4_outlier_b200 as w4

    fused, unfused, Y, Y2 = ffn_setup(synth.FULL_UP, synth.FULL_DOWN, device)
    for _ in range(warmup):
        fused()
        unfused()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [[mk() for _ in range(4)] for _ in range(steps)]
    u_evs = [(mk(), mk()) for _ in range(steps)]
    torch.cuda.synchronize()
    for k in range(steps):
        fused(evs[k])
    for k in range(steps):
        u_evs[k][0].record()
        unfused()
        u_evs[k][1].record()
    torch.cuda.synchronize()
    st, bits = w4.last_error()
    if st != w4.OK:
        raise RuntimeError(f"device error word {bits:#x} in the FFN context")
    avg = lambda i, j: sum(e[i].elapsed_time(e[j]) for e in evs) / steps
    fused_ms = avg(0, 3)
    unfused_ms = sum(a.elapsed_time(b) for a, b in u_evs) / steps
    return {"workload": "ffn: T=57600 5120->13824 k=32 alpha=0.6, GELU, 13824->5120 k=64 alpha=0.7, 32x1",
            "steps": steps, "fused_ms": round(fused_ms, 4),
            "prep_ms": round(avg(0, 1), 4), "up_gemm_fused_ms": round(avg(1, 2), 4),
            "down_gemm_ms": round(avg(2, 3), 4), "unfused_ms": round(unfused_ms, 4),
            "fused_speedup": round(unfused_ms / fused_ms, 3),
            "outputs_bit_identical": bool(torch.equal(Y.view(torch.int16), Y2.view(torch.int16))),
            "note": "online FFN forward (packed weights prepared before timing), timed after the "
                    "headline measurements; bench.py --workload ffn gives the full line"}


def run_ffn(args):
    """The FFN pair at T=57600 ("ffn"; "ffn_mid": T=16384) (Wan2.2 block: 5120 -> 13824, GELU, 13824 -> 5120)
    with the down layer fed by the up layer's output.  Both layers are
    calibrated and packed before the timed region; a step is the online
    forward of one batch: fused (prep, up GEMM whose epilogue writes the down
    layer's quantised activations, down GEMM) and, timed after it for
    comparison, unfused (up linear to bf16 Y, GELU, down linear)."""
    import torch

    import synth
    import w4a4_mxfp4_outlier_b200 as w4

    world, rank, local = dist_env()
    check_device(local)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    active = dist_init("nccl", world, rank)
    Lu, Ld = synth.FULL_UP.with_(seed=1000 * rank), synth.FULL_DOWN
    if args.workload == "ffn_mid":            # the same pair at T=16384 (profiling size)
        Lu = synth.MID_UP.with_(seed=1000 * rank)
    T, d_model, d_ff = Lu.T, Lu.d_in, Lu.d_out
    fused, unfused, Y, Y2 = ffn_setup(Lu, Ld, device, rank)
    mk = lambda: torch.cuda.Event(enable_timing=True)

    for _ in range(args.warmup):
        fused()
        unfused()
    st, bits = w4.last_error()
    if st != w4.OK:
        raise RuntimeError(f"device error word {bits:#x} during warm-up")
    if not torch.equal(Y.view(torch.int16), Y2.view(torch.int16)):
        raise RuntimeError("fused and unfused FFN outputs differ")

    evs = [[mk() for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = mk(), mk()
    u_evs = [(mk(), mk()) for _ in range(args.steps)]
    flush = l2_flush_buffer(ffn_input_bytes(Lu), device)
    clocks = clock_sampler(local)
    torch.cuda.synchronize()
    dist_barrier(active, device)
    clocks.start()
    time.sleep(0.2)
    clocks.mark_start()
    t0.record()
    launches = 0
    for k in range(args.steps):
        if flush is not None:
            flush.zero_()                       # between steps, outside the step's events
        launches += fused(evs[k])
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    clock_info = clocks.stop()
    for k in range(args.steps):
        if flush is not None:
            flush.zero_()
        u_evs[k][0].record()
        unfused()
        u_evs[k][1].record()
    torch.cuda.synchronize()
    dist_barrier(active, device)
    step_ms = sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps
    step_ms_max = dist_max(step_ms, active, device)
    unfused_ms = sum(a.elapsed_time(b) for a, b in u_evs) / args.steps
    flops = 2.0 * (2.0 * T * d_model * d_ff)
    value = aggregate(flops, world, step_ms_max * 1e-3) / 1e12
    avg = lambda i, j: sum(e[i].elapsed_time(e[j]) for e in evs) / args.steps
    prep_ms, up_ms, down_ms = avg(0, 1), avg(1, 2), avg(2, 3)
    gemm_tflops = flops / ((up_ms + down_ms) * 1e-3) / 1e12
    peaks, src = measured_peaks()
    key, _ = peak_keys(step_ms * args.steps * 1e-3)
    fp4_peak = peaks[key] * FP4_PER_BF16
    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1/e8m0 x e2m1/e8m0 + bf16 x bf16, f32 accumulate",
            "data": "synthetic (seeded heavy-tailed X, clipped-normal W; see synth/)",
            "config": ffn_workload_config(args.workload, Lu, Ld, world, flush is not None),
            "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1),
                         "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                         "frac": round(gemm_tflops / fp4_peak, 4), "traffic": None,
                         "kernel": "gemm_dual_pair_kernel (up with fused epilogue, down)",
                         "peak_source": f"{src}: {key} x {FP4_PER_BF16:g}, of measured"},
            "cpu_baseline": None,
            "e2e": None,
            "gpu_launches": launches,
            "clocks": clock_info,
            "kernels": {"prep_ms": round(prep_ms, 4), "up_gemm_fused_ms": round(up_ms, 4),
                        "down_gemm_ms": round(down_ms, 4), "gemm_tflops": round(gemm_tflops, 1),
                        "unfused_ms_per_step": round(unfused_ms, 4),
                        "fused_speedup": round(unfused_ms / step_ms, 3),
                        "outputs_bit_identical": True},
        }
        print(json.dumps(out), flush=True)
    if active:
        import torch.distributed as dist
        dist.destroy_process_group()


def free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def self_launch_cmd(argv, n: int, port: int):
    """The command that runs this script on n ranks of one node: torch's own
    launcher (one process per GPU, RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*
    set for each), rendezvous on 127.0.0.1, the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="full",
                    choices=["full", "full_up", "full_down", "mid_up", "mid_down", "ffn0", "ffn2", "tiny",
                             "sweep", "ffn", "ffn_mid"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ffn-context", action="store_true",
                    help="skip the FFN pair (fused against unfused) timed after the headline line")
    ap.add_argument("--report", action="store_true",
                    help="one JSON line per workload configuration (tiny, ffn0, ffn2, the two "
                         "full layers, every sweep point) instead of the headline line")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)      # at least three untimed warm-up steps
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # launched as `bench.py --gpus N`: start the N ranks here, one per GPU,
        # and return the launcher's status (each rank re-enters with WORLD_SIZE set)
        return subprocess.call(self_launch_cmd(argv, args.gpus, free_port()))
    world = dist_env()[0]
    if world != args.gpus and world > 1:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; running {world} ranks",
              file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.report:
        run_report(args)
    elif args.workload in ("ffn", "ffn_mid"):
        run_ffn(args)
    else:
        run_gpu(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
