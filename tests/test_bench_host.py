"""Host-side logic of bench.py (no GPU): the algorithmic FLOP / byte counts
the roofline divides by, the clock summary, the JSON contract's guards, and
the max-over-ranks reduction on a 2-rank gloo group."""
import json
import multiprocessing as mp
import os
import socket

import pytest

import bench


def test_prefill_work_matches_the_stated_figures():
    # 4Bd + 4d^2 = 196,608 FLOPs per (token, head) at B=256, d=128
    f = bench.prefill_flops(1, 1, 1, 128, 256)
    assert f["formula"] == 196608
    assert f["causal"] == 2 * 257 * 128 + 4 * 128 * 128
    big = bench.prefill_flops(1, 64, 131072, 128, 256)
    assert abs(big["formula"] - 1.649e12) / 1.649e12 < 1e-3
    # q, k, v, o in bf16 + fp32 state out: 8.594 GB for the long-context case
    by = bench.prefill_bytes(1, 64, 131072, 128, 2, state_in=False, state_out=True)
    assert abs(by - 8.594e9) / 8.594e9 < 1e-3


def test_config_states_the_bytes_a_step_streams():
    from linear_attention_lightning_b200 import inputs
    c = bench.workload_config(inputs.WORKLOADS["m1_prefill_128k"], 1)
    assert c["l2"] == "inputs larger than L2 (8.6 GB per step)"  # bf16 q, k, v, o + fp32 state
    assert c["parallelism"] == "single GPU"
    assert bench.workload_config(inputs.WORKLOADS["m1_prefill_128k"], 4)["parallelism"] == "replicas"


def test_long_tensor_bound_legs_are_held_to_the_sustained_peak():
    peaks = {"bf16_tflops": 1656.8, "bf16_tflops_sustained": 1388.7}
    assert bench.tensor_peak(peaks, 0.72) == (1388.7, "sustained")   # 3 steps of 240 ms
    assert bench.tensor_peak(peaks, 0.036) == (1656.8, "burst")      # 20 steps of 1.8 ms


def test_decode_bytes():
    # state read + written (2 * 4 * d^2) plus four bf16 vectors per (seq, head)
    assert bench.decode_bytes(1, 1, 128) == 2 * 4 * 128 * 128 + 4 * 128 * 2
    assert abs(bench.decode_bytes(64, 64, 128) - 541.1e6) / 541.1e6 < 1e-3


def test_roofline_fraction():
    r = bench.roofline("hbm", 3260.1, 6520.2, "GB/s", None)
    assert r["frac"] == 0.5 and r["bound"] == "hbm" and r["traffic"] is None


def test_clock_summary_flags_throttling():
    rows = [{"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "power_w": 800.0, "hw_slowdown": "Not Active",
             "hw_thermal_slowdown": "Not Active", "sw_thermal_slowdown": "Not Active",
             "sw_power_cap": "Active"},
            {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "power_w": 900.0, "hw_slowdown": "Not Active",
             "hw_thermal_slowdown": "Active", "sw_thermal_slowdown": "Not Active",
             "sw_power_cap": "Not Active"},
            {"sm_mhz": 300.0, "sm_max_mhz": 1965.0, "power_w": 90.0, "hw_slowdown": "Not Active",
             "hw_thermal_slowdown": "Not Active", "sw_thermal_slowdown": "Not Active",
             "sw_power_cap": "Not Active"}]
    c = bench.summarize_clocks(rows)
    assert c["sm_mhz"] == 1850.0            # idle sample excluded
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.summarize_clocks([])["sm_mhz"] is None


def test_warmup_floor():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.impl == "ours"


def test_stored_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    import shutil
    shutil.copytree(os.path.join(bench.ROOT, "linear_attention_lightning_b200", "csrc"),
                    tmp_path / "linear_attention_lightning_b200" / "csrc")
    shutil.copytree(os.path.join(bench.ROOT, "include"), tmp_path / "include")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    prof = tmp_path / "profiles"
    prof.mkdir()

    def store():
        (prof / "traffic.json").write_text(json.dumps({"launches": {
            "w/pair": {"kernel_source_digest": bench.kernel_source_digest("prefill_pair.cuh"),
                       "dram_bytes_per_launch": 123},
            "w/norm_gate": {"kernel_source_digest": bench.kernel_source_digest("norm_gate.cuh"),
                            "dram_bytes_per_launch": 456}}}))

    store()
    assert bench.measured_traffic("w", "pair") == 123
    assert bench.measured_traffic("w", "norm_gate") == 456
    assert bench.measured_traffic("w", "decode") is None  # never captured
    csrc = tmp_path / "linear_attention_lightning_b200" / "csrc"
    # a change to one kernel voids its own counters only
    with open(csrc / "norm_gate.cuh", "a") as f:
        f.write("// edit\n")
    assert bench.measured_traffic("w", "norm_gate") is None
    assert bench.measured_traffic("w", "pair") == 123
    # a change to a shared header voids every kernel that includes it
    store()
    with open(csrc / "common.cuh", "a") as f:
        f.write("// edit\n")
    assert bench.measured_traffic("w", "pair") is None
    assert bench.measured_traffic("w", "norm_gate") is None
    # the public header (declarations only) is not part of any kernel's sources
    store()
    with open(tmp_path / "include" / "lightning.h", "a") as f:
        f.write("// edit\n")
    assert bench.measured_traffic("w", "pair") == 123
    assert bench.measured_traffic("w", "norm_gate") == 456


def _rank_main(rank, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, world, _ = bench.dist_setup(2)
    bench.barrier(world)
    got = bench.max_over_ranks(10.0 + r, world)
    q.put((r, world, got))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 2, 11.0), (1, 2, 11.0)]


def test_every_stored_traffic_entry_names_a_known_kernel():
    # each stored counter is looked up by (workload, kernel) and checked against that
    # kernel's source digest, so its kernel must be one bench.py knows the header of
    stored = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))["launches"]
    assert stored
    for key, entry in stored.items():
        workload, _, kernel = key.partition("/")
        assert workload and kernel in bench.KERNEL_SOURCES, key
        assert len(entry["kernel_source_digest"]) == 16, key
        assert any(f in entry for f in ("dram_bytes_per_launch", "dram_bytes_per_step")), key


class _FakeNvml:
    """Stands in for pynvml: one GPU at bus 00000000:1B:00.0, SM clock 1965 of 1965 MHz,
    800 W, the power cap the only active clock-event reason. Records what it is asked."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    def __init__(self, fail_init=False):
        self.fail_init, self.calls, self.inited = fail_init, [], 0

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no driver")
        self.inited += 1

    def nvmlShutdown(self):
        self.inited -= 1

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self.calls.append(("bus", bus))
        return "gpu"

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append(("index", i))
        return "gpu"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 800000

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 | 0x1  # power cap, plus a reason the bench does not report (idle)


def test_clock_sampler_reads_nvml_over_the_timed_region():
    import time
    nv = _FakeNvml()
    with bench.ClockSampler(0, bus_id="00000000:1B:00.0", nvml=nv) as clk:
        time.sleep(0.03)
    s = clk.summary()
    assert ("bus", "00000000:1B:00.0") in nv.calls and nv.inited == 0
    assert s["source"].startswith("nvml") and s["samples"] >= 3
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_falls_back_when_nvml_is_unavailable():
    nv = _FakeNvml(fail_init=True)
    with bench.ClockSampler(0, nvml=nv) as clk:
        pass
    s = clk.summary()
    assert s["source"].startswith("nvidia-smi") and not clk.poller.ok
    # no nvidia-smi on a host without a GPU either: reported as not sampled, not invented
    if not clk.rows:
        assert s["reasons"] == ["not sampled"] and s["sm_mhz"] is None


def test_reference_arm_prints_one_contract_line_on_rank_zero_only():
    # the reference arm times the oracle on the host cores: one JSON line with the
    # contract's keys on rank 0, nothing (and exit 0) on the other ranks
    import subprocess
    import sys
    cmd = [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
           "--warmup", "3"]
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=bench.ROOT)
    assert r.returncode == 0 and r.stdout.strip() == "", r.stderr[-500:]
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE")}
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-500:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["steps"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == bench.PREFILL_WORKLOAD
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


class _FakeAbi:
    """Stands in for the binding: a status word that reads `status` once."""
    LA_OK, LA_ERR_TIMEOUT = 0, 4

    def __init__(self, status):
        self.status, self.asked = status, 0

    def lightning_last_device_status(self, stream):
        self.asked += 1
        return self.status

    def status_string(self, st):
        return {0: "LA_OK", 4: "LA_ERR_TIMEOUT: a device-side wait gave up"}[st]


def test_a_leg_whose_kernels_recorded_a_failure_is_not_a_measurement():
    # a kernel whose bounded wait ran out returns early: its time would read as a fast step
    ok = _FakeAbi(0)
    bench.check_device_status("decode", ok, 0, 1)
    assert ok.asked == 1
    with pytest.raises(bench.LegFailed, match="decode: a kernel recorded LA_ERR_TIMEOUT"):
        bench.check_device_status("decode", _FakeAbi(4), 0, 1)


def _status_rank_main(rank, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, world, _ = bench.dist_setup(2)
    # only rank 1's kernels recorded a failure; both ranks must fail the leg alike
    try:
        bench.check_device_status("backward", _FakeAbi(4 if r == 1 else 0), 0, world)
        q.put((r, "passed"))
    except bench.LegFailed:
        q.put((r, "failed"))
    bench.barrier(world)   # both ranks are still in step
    import torch.distributed as dist
    dist.destroy_process_group()


def test_a_failure_on_one_rank_fails_the_leg_on_every_rank():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_status_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, "failed"), (1, "failed")]


def test_auxiliary_legs_go_on_lines_of_their_own():
    line = json.loads(bench.aux_line("backward", {"ms_per_step": 1.0}))
    assert line == {"aux": "backward", "result": {"ms_per_step": 1.0}}
