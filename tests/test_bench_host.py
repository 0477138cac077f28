"""Host-side pieces of bench.py on CPU: the multi-rank plumbing over gloo with
world size 2 (barrier, max over ranks, whole-job aggregation) and the
reference arm (the CPU oracle), which only rank 0 runs and prints."""
import io
import json
import multiprocessing as mp
import os
import socket

from contextlib import redirect_stdout

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist
    w, r, _ = bench.dist_env()
    active = bench.dist_init("gloo", w, r, timeout_s=60)
    bench.dist_barrier(active)
    step_s = 0.5 + rank            # rank 1 is the slow one
    m = bench.dist_max(step_s, active, torch.device("cpu"))
    q.put((rank, active, m, bench.aggregate(100.0, w, m)))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for rank, active, m, agg in res:
        assert active and m == 1.5                      # max over ranks
        assert agg == 100.0 * 2 / 1.5                   # all ranks' units / slowest time


def test_single_rank_is_not_distributed():
    assert bench.dist_init("gloo", 1, 0) is False
    assert bench.dist_max(3.0, False, None) == 3.0


def test_reference_arm_prints_on_rank0_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert buf.getvalue() == ""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["warmup"] == 3
    # the same config the GPU arm prints for this workload
    import synth
    assert line["config"] == bench.layer_workload_config("tiny", synth.WORKLOADS["tiny"], 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True





def test_l2_flush_only_where_inputs_fit_in_twice_l2():
    import synth
    flushed = lambda w: bench.layer_workload_config(w, synth.WORKLOADS[w], 1)["l2"].startswith("L2 flushed")
    # X_up alone is 590 MB and X_down 1.6 GB: no flush needed on the full layers
    assert not flushed("full") and not flushed("full_up") and not flushed("full_down")
    assert flushed("tiny")
    # X 168 MB + W 142 MB reach twice the 126 MB L2; the FFN step reads X alone
    assert not bench.layer_input_bytes(synth.MID_UP) < 2 * bench.L2_BYTES
    assert bench.ffn_workload_config("ffn_mid", synth.MID_UP, synth.MID_DOWN, 1)["l2"].startswith("L2 flushed")
    assert bench.l2_flush_buffer(bench.layer_input_bytes(synth.WORKLOADS["full"][0]), None) is None


def test_peak_choice_by_timed_region_length():
    assert bench.peak_keys(0.04) == ("bf16_tflops", "bf16_tflops_sustained")
    assert bench.peak_keys(1.5) == ("bf16_tflops_sustained", "bf16_tflops")


class _FakeNvml:
    """Stands in for pynvml: the clock drops under a power cap from `switch`
    (a time.time() value) on."""
    NVML_CLOCK_SM = 0

    def __init__(self):
        self.switch = float("inf")

    def _capped(self):
        import time
        return time.time() >= self.switch

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        return 1400 if self._capped() else 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 1000000 if self._capped() else 600000        # milliwatts

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 if self._capped() else 0x0               # sw_power_cap


def test_nvml_sampler_summarises_the_timed_window():
    import time
    fake = _FakeNvml()
    s = bench.NvmlClockSampler(object(), fake)
    s.start()
    time.sleep(0.03)
    fake.switch = time.time()
    s.mark_start()
    time.sleep(0.12)
    s.mark_end()
    time.sleep(0.03)
    out = s.stop()
    assert out["source"] == "nvml, 5 ms" and out["samples"] >= 3
    assert out["sm_max_mhz"] == 1965.0 and out["sm_mhz"] == 1400.0 and out["sm_min_mhz"] == 1400.0
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 1000.0
    # samples outside the window are not counted
    assert out["samples"] < len(s.samples)


def test_clock_sampler_without_nvml_or_nvidia_smi():
    s = bench.clock_sampler(0)          # no GPU here: NVML fails, nvidia-smi is absent
    s.start()
    s.mark_start()
    s.mark_end()
    out = s.stop()
    assert out["sm_mhz"] is None and out["reasons"]


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` (no launcher around it) starts two ranks itself;
    rank 0 alone prints the one JSON line, which reports both ranks.  The
    reference arm runs here (CPU), through the same launch path."""
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        "--gpus", "2", "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_self_launch_command():
    cmd = bench.self_launch_cmd(["--gpus", "4", "--steps", "5"], 4, 29512)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29512" in cmd and cmd[-4:] == ["--gpus", "4", "--steps", "5"]
    assert cmd[-5].endswith("bench.py")
