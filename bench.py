"""Benchmark of the Lightning Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one lightning_prefill call over the long-context workload
(batch 1, 64 heads, 131072 tokens, head dim 128, block 256, bf16 q/k/v/o,
fp32 state), inputs resident in HBM. The same run also times the decode
workload (64 sequences x 64 heads x 128, fp32 states, 1000 consecutive
single-token steps) and the end-to-end path with host buffers; these go into
the contract line, which rank 0 prints last. Auxiliary legs (snapshots, the
norm-and-gate epilogue, the softmax GQA layer, the other workloads, the
hybrid block, the backward) come before it, one JSON line each
({"aux": name, "result": ...}). After every timed region the library's status
word is checked on every rank: a leg whose kernels recorded a failure is no
measurement (the prefill and decode legs then end the run; an auxiliary leg
is reported as failed). With --gpus N (under torchrun) every rank runs an
independent replica of the workload ("replicas only": the path has no
exchange step); times are the max over ranks.

`--impl reference` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PREFILL_WORKLOAD = "m1_prefill_128k"
DECODE_WORKLOAD = "batched_decode"
METRIC = "prefill tokens/s & TFLOP/s (% bf16 peak); decode state GB/s (% HBM peak)"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- arithmetic

def prefill_flops(batch, heads, seq, dim, block):
    """Algorithmic FLOPs of one prefill, two conventions, per (token, head):
    formula 4Bd + 4d^2 (dense masked BxB products as the block formula writes
    them, plus the inter and state products); causal 2(B+1)d + 4d^2."""
    units = batch * heads * seq
    return {"formula": units * (4 * block * dim + 4 * dim * dim),
            "causal": units * (2 * (block + 1) * dim + 4 * dim * dim)}


def prefill_bytes(batch, heads, seq, dim, elem_bytes=2, state_in=False, state_out=True):
    """Algorithmic HBM bytes of one prefill: q, k, v read and o written once,
    plus the fp32 states read / written once."""
    tok = 4 * batch * heads * seq * dim * elem_bytes
    st = batch * heads * dim * dim * 4
    return tok + (st if state_in else 0) + (st if state_out else 0)


def decode_bytes(batch, heads, dim, elem_bytes=2):
    """Algorithmic HBM bytes of one decode step: the fp32 state read and
    written once, q, k, v read and o written once."""
    return batch * heads * (2 * dim * dim * 4 + 4 * dim * elem_bytes)


def workload_config(w, world):
    """The contract line's config, the same for both arms: the workload by name
    and sizes, how the run is spread over GPUs, and how L2 is kept out of the
    timing (every step streams more than L2 holds)."""
    by = prefill_bytes(w.batch, w.heads, w.seq, w.dim, 2 if str(w.dtype) == "torch.bfloat16" else 4,
                       state_in=w.state_in, state_out=True)
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "seq_len": w.seq, "dim": w.dim,
            "block": w.block, "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (%.1f GB per step)" % (by / 1e9)}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# A tensor-bound leg whose timed region lasts longer than this is held to the
# sustained bf16 peak (the power cap's clocks); a shorter one to the burst peak.
SUSTAINED_AFTER_S = 0.5


def tensor_peak(peaks, timed_s):
    """(peak TFLOP/s, which one) for a tensor-bound leg timed over timed_s seconds."""
    if timed_s > SUSTAINED_AFTER_S:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def roofline(bound, achieved, peak, unit, traffic=None):
    return {"bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4) if peak else None, "traffic": traffic}


KERNEL_SOURCES = {  # traffic.json key suffix -> the header that holds the kernel
    "pair": "prefill_pair.cuh", "tcgen05": "prefill_tc.cuh", "simt": "prefill_simt.cuh",
    "backward_pair": "prefill_pair.cuh", "decode": "decode.cuh", "norm_gate": "norm_gate.cuh",
    "gqa_partial": "gqa_decode_tc.cuh", "gqp_attn": "gqa_prefill.cuh", "prefill_norm_gate": "prefill_pair.cuh",
}


def kernel_source_digest(header):
    """Digest of one kernel's header and every kernel source it includes (the
    files under csrc/; the public header holds only declarations), to tell
    whether stored ncu counters still describe the kernel being timed."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "linear_attention_lightning_b200", "csrc")
    seen, todo = [], [os.path.normpath(os.path.join(csrc, header))]
    while todo:
        path = todo.pop()
        if path in seen or os.path.dirname(path) != os.path.normpath(csrc):
            continue
        seen.append(path)
        with open(path, "rb") as f:
            text = f.read()
        for inc in re.findall(rb'#include "([^"]+)"', text):
            todo.append(os.path.normpath(os.path.join(os.path.dirname(path), inc.decode())))
    h = hashlib.sha256()
    for path in sorted(seen):
        with open(path, "rb") as f:
            h.update(os.path.relpath(path, ROOT).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, kernel, field="dram_bytes_per_launch"):
    """DRAM bytes from the committed ncu summary, or None when the kernel's
    sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get("launches", {}).get("%s/%s" % (workload, kernel))
    if entry is None or entry.get("kernel_source_digest") != kernel_source_digest(KERNEL_SOURCES[kernel]):
        return None
    return entry.get(field)


def summarize_clocks(rows):
    """rows: list of dicts from nvidia-smi samples; returns the clocks object."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["not sampled"]}
    loaded = [r for r in rows if r.get("power_w", 0) > 200] or rows
    sm = statistics.median(r["sm_mhz"] for r in loaded)
    reasons = set()
    for r in loaded:
        for key in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"):
            if r.get(key) == "Active":
                reasons.add(key)
    return {"sm_mhz": sm, "sm_max_mhz": max(r["sm_max_mhz"] for r in rows),
            "reasons": sorted(reasons), "samples": len(loaded)}


class NvmlPoller:
    """Reads one GPU's SM clock, power draw and clock-event reasons through NVML every
    `period` seconds from a thread, in the rows summarize_clocks takes. Queries only: no
    setting of the GPU is changed. A timed region of tens of milliseconds falls between
    the samples of nvidia-smi's 200 ms loop; this one lands several inside it. Any NVML
    failure leaves it empty (ok False), and the caller falls back to nvidia-smi."""

    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"))

    def __init__(self, bus_id=None, index=0, period=0.002, nvml=None):
        self.bus_id, self.index, self.period, self.nv = bus_id, index, period, nvml
        self.rows = []
        self.ok = False
        self._stop = threading.Event()
        self._thread = None
        self._sample = None

    def start(self):
        try:
            nv = self.nv
            if nv is None:
                import pynvml as nv
                self.nv = nv
            nv.nvmlInit()
            self.ok = True  # initialised: stop() shuts NVML down again
            h = (nv.nvmlDeviceGetHandleByPciBusId(self.bus_id) if self.bus_id
                 else nv.nvmlDeviceGetHandleByIndex(self.index))
            reasons = (getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None)
                       or nv.nvmlDeviceGetCurrentClocksThrottleReasons)
            bits = {name: (getattr(nv, "nvmlClocksEventReason" + suffix, None)
                           or getattr(nv, "nvmlClocksThrottleReason" + suffix)) for name, suffix in self.REASONS}
            sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def sample():
                r = int(reasons(h))
                row = {"sm_mhz": float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), "sm_max_mhz": sm_max,
                       "power_w": nv.nvmlDeviceGetPowerUsage(h) / 1000.0}
                for name, bit in bits.items():
                    row[name] = "Active" if r & int(bit) else "Not Active"
                return row

            sample()  # a query that is not available fails here, before the thread starts
            self._sample = sample
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self.stop()
            self.ok = False
        return self

    def _run(self):
        while not self._stop.is_set():
            try:
                self.rows.append(self._sample())
            except Exception:
                return
            self._stop.wait(self.period)

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)
            self._thread = None
        if self.ok and self.nv is not None:
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass


def pci_bus_id_of(dev):
    """The PCI bus id of a torch CUDA device ("00000000:1B:00.0"), or None: NVML's
    device order need not follow CUDA_VISIBLE_DEVICES, the bus id does not depend on it."""
    try:
        import torch
        p = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


class ClockSampler:
    """Samples clocks and throttle reasons while the timed region runs: NVML every 2 ms
    (NvmlPoller), with nvidia-smi's loop as the fallback when NVML is not available."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, bus_id=None, nvml=None):
        self.gpu_index = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None
        self.poller = NvmlPoller(bus_id=bus_id, index=gpu_index, nvml=nvml)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        self.poller.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                self.rows.append({"sm_mhz": float(parts[0]), "sm_max_mhz": float(parts[1]),
                                  "power_w": float(parts[2]), "hw_slowdown": parts[3],
                                  "hw_thermal_slowdown": parts[4], "sw_thermal_slowdown": parts[5],
                                  "sw_power_cap": parts[6]})
            except ValueError:
                continue

    def __exit__(self, *exc):
        self.poller.stop()  # at the end of the timed region
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=5)
        return False

    def summary(self):
        if len(self.poller.rows) >= 3:
            out = summarize_clocks(self.poller.rows)
            out["source"] = "nvml every 2 ms over the timed region"
        else:
            out = summarize_clocks(self.rows)
            out["source"] = "nvidia-smi -lms 200"
        return out


# ---------------------------------------------------------------- ranks

def dist_setup(n_gpus):
    """Returns (rank, world, local_rank). Initialises torch.distributed when launched by torchrun."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist.get_rank(), world, int(os.environ.get("LOCAL_RANK", "0"))
    return 0, 1, 0


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cpu"):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class LegFailed(RuntimeError):
    """A timed leg whose kernels recorded a failure in the status word."""


def check_device_status(leg, abi, stream_handle, world, device="cpu"):
    """After a timed region: the library's status word must be clean on every
    rank. A kernel whose bounded wait ran out returns early, and its time would
    read as a fast step, so such a leg is no measurement. Collective (every
    rank takes the same step), then raises on every rank if any rank failed."""
    st = abi.lightning_last_device_status(stream_handle)
    worst = max_over_ranks(0.0 if st == abi.LA_OK else float(st), world, device)
    if worst:
        raise LegFailed("%s: a kernel recorded %s during the timed region" % (leg, abi.status_string(int(worst))))


def timed(leg, step, steps, warmup, stream, world, device):
    """`warmup` untimed calls, then `steps` calls between CUDA events on
    `stream`, bracketed by a barrier and a synchronisation; the status word is
    checked afterwards. Returns milliseconds per step, the max over ranks."""
    import torch
    from linear_attention_lightning_b200 import abi
    for _ in range(warmup):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, device) / steps
    check_device_status(leg, abi, stream.cuda_stream, world, device)
    return ms


def aux_line(name, result):
    """One auxiliary leg's result as its own JSON line, printed before the
    contract line so that the contract line stays short."""
    return json.dumps({"aux": name, "result": result})


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(w, tokens, heads, threads=None, h0=0):
    """Time the float64 oracle (token recurrence) on `heads` heads (from head
    h0) x `tokens` tokens of the workload's distribution; returns (seconds,
    token-heads)."""
    import numpy as np
    import oracle
    from linear_attention_lightning_b200 import inputs
    if threads:
        oracle.set_threads(threads)
    inp = inputs.prefill_inputs(1, heads, tokens, w.dim, w.dtype, w.state_in, seed=w.seed + h0)
    conv = inputs.to_oracle
    sl = inputs.slopes(w.heads)[h0:h0 + heads].numpy()
    args = (conv(inp["q"]), conv(inp["k"]), conv(inp["v"]), sl, None)
    t0 = time.perf_counter()
    oracle.prefill(*args, form="recurrence")
    return time.perf_counter() - t0, tokens * heads


def cpu_baseline(w, budget_s=25.0):
    """The oracle on a bounded sample of the workload, sized to about budget_s
    of CPU work: groups of up to one head per core (inputs and the float64
    output of a whole head group stay a few GB), each up to the full sequence."""
    import oracle
    cores = oracle.threads()
    heads = min(w.heads, max(1, cores))
    sec, units = oracle_sample(w, 2048, heads)
    rate = units / max(sec, 1e-6)                               # token-heads per second
    want = rate * budget_s * 0.8
    tokens = int(min(w.seq, max(2048, want / heads)))
    groups = int(max(1, min(w.heads // heads, round(want / (heads * tokens)))))
    sec = units = 0
    for g in range(groups):
        s_g, u_g = oracle_sample(w, tokens, heads, h0=g * heads)
        sec += s_g
        units += u_g
    tok_per_s = units / w.heads / sec  # a token covers every head
    return {"value": round(tok_per_s, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "float64 token recurrence, %d of %d heads x %d tokens of the %s workload, %.1f s"
                      % (heads * groups, w.heads, tokens, w.name, sec)}


def run_reference(args):
    # rank 0 alone runs the CPU oracle; the other ranks exit without work
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from linear_attention_lightning_b200 import inputs
    w = inputs.WORKLOADS[PREFILL_WORKLOAD]
    import oracle
    cores = oracle.threads()
    heads = min(w.heads, max(1, cores))
    budget = 150.0 / max(1, args.steps + args.warmup)
    sec, units = oracle_sample(w, 1024, heads)
    tokens = int(min(w.seq, max(1024, 1024 * budget / max(sec, 1e-3) * 0.7)))
    for _ in range(args.warmup):
        oracle_sample(w, min(tokens, 1024), heads)
    times = []
    for _ in range(args.steps):
        sec, units = oracle_sample(w, tokens, heads)
        times.append(sec)
    tot = sum(times)
    value = args.steps * units / w.heads / tot
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * tot / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world), "inputs": "bf16 q,k,v widened to float64",
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": "%d of %d heads x %d tokens per step" % (heads, w.heads, tokens)},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU path

def run_ours(args):
    import torch
    import linear_attention_lightning_b200 as la
    from linear_attention_lightning_b200 import abi, inputs

    rank, world, local_rank = dist_setup(args.gpus)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    w = inputs.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    inp = inputs.workload_inputs(w, dev)
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    o = torch.empty_like(q)
    s_out = torch.empty((w.batch, w.heads, w.dim, w.dim), dtype=torch.float32, device=dev)
    # the main leg may time another block length or kernel than the library picks
    # for the workload (--block, --variant); the other legs keep the workload's own
    wm = dataclasses.replace(w, block=args.block) if args.block else w
    variant = (la.prefill_variant(wm.dtype, wm.batch, wm.heads, wm.seq, wm.dim, wm.block) if args.variant == "auto"
               else args.variant)
    vcode = {"simt": abi.LA_VARIANT_SIMT, "tcgen05": abi.LA_VARIANT_TCGEN05,
             "pair": abi.LA_VARIANT_TCGEN05_PAIR}[variant]
    dcode = abi.LA_DTYPE_BF16 if w.dtype == torch.bfloat16 else abi.LA_DTYPE_F32
    # kernels one lightning_prefill_ex call launches: a tensor-core kernel, then its
    # range guard's second pass (which returns at once for heads it need not redo)
    launches_per_step = 2 if variant in ("pair", "tcgen05") else 1
    need = abi.lightning_prefill_workspace_size(wm.batch, wm.heads, wm.seq, wm.dim, wm.block)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def step():
        abi.check(abi.lightning_prefill_ex(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), dcode, sl.data_ptr(), wm.batch, wm.heads,
            wm.seq, wm.dim, wm.block, None if s0 is None else s0.data_ptr(), o.data_ptr(),
            s_out.data_ptr(), ws.data_ptr(), need, sp, vcode))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank, bus_id=pci_bus_id_of(dev)) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    per_launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    check_device_status("prefill", abi, sp, world, dev)
    ms_per_step = total_ms / args.steps
    tokens = w.batch * w.seq
    value = world * tokens * args.steps / (total_ms / 1e3)

    fl = prefill_flops(wm.batch, wm.heads, wm.seq, wm.dim, wm.block)
    by = prefill_bytes(wm.batch, wm.heads, wm.seq, wm.dim, 2 if wm.dtype == torch.bfloat16 else 4,
                       state_in=s0 is not None, state_out=True)
    avg_launch_s = statistics.mean(per_launch_ms) / 1e3
    gbs = by / avg_launch_s / 1e9
    tflops = {kk: vv / avg_launch_s / 1e12 for kk, vv in fl.items()}
    traffic = measured_traffic(w.name, variant) if wm.block == w.block else None

    # decode: 1000 consecutive single-token steps over fp32 states
    dw = inputs.WORKLOADS[DECODE_WORKLOAD]
    dec = run_decode(dw, dev, stream, peaks, args, world) if args.decode_steps > 0 else None

    # end to end: host buffers, copies inside the timed region
    e2e = run_e2e(w, dev, stream, inp, variant, args, world) if args.e2e_steps > 0 else None

    # Auxiliary legs, each printed on a line of its own before the contract line.
    # A leg whose kernels recorded a failure is reported as failed (on every rank
    # alike) and the run goes on; the contract line lists the failed legs.
    failed = []

    def aux(name, enabled, fn):
        if not enabled:
            return
        try:
            r = fn()
        except LegFailed as exc:
            failed.append(name)
            r = {"failed": str(exc)}
        if rank == 0:
            print(aux_line(name, r), flush=True)

    # the same prefill keeping prefix-cache snapshots of the state
    aux("snapshots", args.snapshot_interval > 0 and w.seq >= args.snapshot_interval,
        lambda: run_snapshots(w, dev, stream, inp, vcode, dcode, args, world, ms_per_step))
    # normalisation and gating of the prefill's output
    aux("norm_gate", args.norm_gate_steps > 0, lambda: run_norm_gate_leg(w, dev, stream, o, dcode, args, world))
    # the same prefill with the per-head normalisation and gate fused into its epilogue
    aux("prefill_norm_gate", args.fused_norm_gate_steps > 0 and variant == "pair",
        lambda: run_prefill_norm_gate_leg(w, dev, stream, inp, dcode, args, world))
    # decode step and prefill of the softmax GQA layer the hybrid model interleaves
    aux("gqa_decode", args.gqa_steps > 0, lambda: run_gqa_leg(dev, stream, args, world))
    aux("gqa_prefill", args.gqa_prefill_steps > 0, lambda: run_gqa_prefill_leg(dev, stream, args, world))
    # the other prefill workloads: many short sequences with carried-in states; 8192 tokens
    for n in ("batched_prefill_state", "m1_prefill_8k"):
        aux("other_workloads/" + n, args.batched_steps > 0 and n != w.name,
            lambda n=n: run_workload_leg(n, dev, stream, peaks, args, world))
    # one block of the hybrid model's attention: 7 Lightning layers and 1 softmax layer
    aux("hybrid_block", args.hybrid_steps > 0 and w.dtype == torch.bfloat16 and w.dim == 128,
        lambda: run_hybrid_leg(w, dev, stream, inp, vcode, dcode, args, world))
    aux("hybrid_decode", args.hybrid_steps > 0 and args.gqa_steps > 0,
        lambda: run_hybrid_decode_leg(dev, stream, args, world))
    # gradients of the same prefill (dq, dk, dv, d state_in)
    aux("backward", args.backward_steps > 0, lambda: run_backward_leg(w, dev, stream, inp, dcode, args, world))

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wm, world),
        "kernel": variant,
        "tflops": {"formula": round(tflops["formula"], 2), "causal": round(tflops["causal"], 2),
                   "peak_bf16": peaks["bf16_tflops"],
                   "frac_formula": round(tflops["formula"] / peaks["bf16_tflops"], 4),
                   "frac_causal": round(tflops["causal"] / peaks["bf16_tflops"], 4),
                   "peak_source": peaks["source"]},
        "roofline": roofline("hbm", gbs, peaks["hbm_gbs"], "GB/s", traffic),
        "decode": dec,
        "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step,
        "aux_legs_failed": failed,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_decode(dw, dev, stream, peaks, args, world=1):
    import torch
    from linear_attention_lightning_b200 import abi, inputs
    steps = args.decode_steps
    inp = inputs.workload_inputs(dw, dev, steps=max(steps, 3))  # 3 warm-up tokens at least
    state = inp["state"]
    qs, ks, vs, sl = inp["q"], inp["k"], inp["v"], inp["slopes"]
    o = torch.empty((dw.batch, dw.heads, dw.dim), dtype=dw.dtype, device=dev)
    sp = stream.cuda_stream
    dcode = abi.LA_DTYPE_BF16
    tok = dw.batch * dw.heads * dw.dim

    def one(t):
        abi.check(abi.lightning_decode(qs[t].data_ptr(), ks[t].data_ptr(), vs[t].data_ptr(), dcode,
                                       sl.data_ptr(), dw.batch, dw.heads, dw.dim, state.data_ptr(),
                                       o.data_ptr(), sp))

    for t in range(3):
        one(t)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for t in range(steps):
        one(t)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    check_device_status("decode", abi, sp, world, dev)
    by = decode_bytes(dw.batch, dw.heads, dw.dim)
    gbs = by * steps / (ms / 1e3) / 1e9
    del tok
    return {"workload": dw.name, "steps": steps, "us_per_step": round(1e3 * ms / steps, 3),
            "value": round(gbs, 1), "unit": "GB/s (state + token bytes)",
            "roofline": roofline("hbm", gbs, peaks["hbm_gbs"], "GB/s", measured_traffic(dw.name, "decode")),
            "l2": "state 268 MB > L2; consecutive steps, no flush"}


def run_snapshots(w, dev, stream, inp, vcode, dcode, args, world, plain_ms):
    """The prefill step through lightning_prefill_snapshots: a state snapshot
    every args.snapshot_interval tokens, timed like the main leg."""
    import torch
    from linear_attention_lightning_b200 import abi
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    interval = args.snapshot_interval
    n = abi.lightning_prefill_snapshot_count(w.seq, interval)
    o = torch.empty_like(q)
    s_out = torch.empty((w.batch, w.heads, w.dim, w.dim), dtype=torch.float32, device=dev)
    snaps = torch.empty((w.batch, w.heads, n, w.dim, w.dim), dtype=torch.float32, device=dev)
    need = abi.lightning_prefill_workspace_size(w.batch, w.heads, w.seq, w.dim, w.block)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_prefill_snapshots(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), dcode, sl.data_ptr(), w.batch, w.heads, w.seq, w.dim,
            w.block, None if s0 is None else s0.data_ptr(), o.data_ptr(), s_out.data_ptr(), interval,
            snaps.data_ptr(), ws.data_ptr(), need, sp, vcode))

    steps = max(1, min(args.steps, 10))
    ms = timed("snapshots", step, steps, args.warmup, stream, world, dev)
    return {"interval": interval, "count": n, "steps": steps, "ms_per_step": round(ms, 4),
            "overhead_vs_plain_pct": round(100.0 * (ms / plain_ms - 1.0), 2),
            "snapshot_bytes_per_step": int(snaps.numel() * 4)}


def run_norm_gate_leg(w, dev, stream, o, dcode, args, world):
    """lightning_norm_gate on the prefill's output: RMS over each token's
    heads*dim channels, sigmoid gate; timed like the main leg."""
    import torch
    from linear_attention_lightning_b200 import abi
    g = torch.Generator(device=dev).manual_seed(w.seed + 2000)
    gate = torch.randn((w.batch, w.seq, w.heads * w.dim), generator=g, device=dev).to(o.dtype)
    gamma = torch.ones(w.heads * w.dim, device=dev)
    y = torch.empty((w.batch, w.seq, w.heads * w.dim), dtype=o.dtype, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_norm_gate(o.data_ptr(), gate.data_ptr(), dcode, gamma.data_ptr(), 1e-6, w.batch,
                                          w.heads, w.seq, w.dim, 0, y.data_ptr(), sp))

    steps = args.norm_gate_steps
    ms = timed("norm_gate", step, steps, args.warmup, stream, world, dev)
    by = 3 * o.numel() * o.element_size() + gamma.numel() * 4  # o, gate read; y written
    gbs = by / (ms / 1e3) / 1e9
    return {"steps": steps, "ms_per_step": round(ms, 4), "per": "token (heads*dim channels)",
            "tokens_per_s": round(world * w.batch * w.seq / (ms / 1e3), 1),
            "roofline": roofline("hbm", gbs, load_peaks()["hbm_gbs"], "GB/s", measured_traffic(w.name, "norm_gate"))}


def run_prefill_norm_gate_leg(w, dev, stream, inp, dcode, args, world):
    """lightning_prefill_norm_gate (the per-head normalisation and gate fused into
    the prefill's epilogue, o never written) against the two calls it replaces
    (lightning_prefill_ex, then lightning_norm_gate with the per-head mean),
    alternating, each timed like the main leg."""
    import torch
    from linear_attention_lightning_b200 import abi
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    g = torch.Generator(device=dev).manual_seed(w.seed + 2000)
    gate = torch.randn((w.batch, w.seq, w.heads * w.dim), generator=g, device=dev).to(q.dtype)
    gamma = torch.ones(w.heads * w.dim, device=dev)
    y = torch.empty((w.batch, w.seq, w.heads * w.dim), dtype=q.dtype, device=dev)
    o = torch.empty_like(q)
    s_out = torch.empty((w.batch, w.heads, w.dim, w.dim), dtype=torch.float32, device=dev)
    sp = stream.cuda_stream
    s0p = None if s0 is None else s0.data_ptr()
    need = abi.lightning_prefill_workspace_size(w.batch, w.heads, w.seq, w.dim, w.block)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def fused():
        abi.check(abi.lightning_prefill_norm_gate(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), dcode, sl.data_ptr(), w.batch, w.heads, w.seq, w.dim,
            w.block, s0p, gate.data_ptr(), gamma.data_ptr(), 1e-6, y.data_ptr(), s_out.data_ptr(), ws.data_ptr(),
            need, sp))

    def two_calls():
        abi.check(abi.lightning_prefill_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), dcode, sl.data_ptr(), w.batch,
                                           w.heads, w.seq, w.dim, w.block, s0p, o.data_ptr(), s_out.data_ptr(),
                                           ws.data_ptr(), need, sp, abi.LA_VARIANT_TCGEN05_PAIR))
        abi.check(abi.lightning_norm_gate(o.data_ptr(), gate.data_ptr(), dcode, gamma.data_ptr(), 1e-6, w.batch,
                                          w.heads, w.seq, w.dim, 1, y.data_ptr(), sp))

    steps = max(1, min(args.fused_norm_gate_steps, 10))
    f_ms, t_ms = [], []
    for _ in range(2):
        f_ms.append(timed("prefill_norm_gate", fused, steps, args.warmup, stream, world, dev))
        t_ms.append(timed("prefill_norm_gate/two_calls", two_calls, steps, args.warmup, stream, world, dev))
    ms, ms2 = min(f_ms), min(t_ms)
    n = q.numel() * q.element_size()
    by = 5 * n + gamma.numel() * 4 + (0 if s0 is None else 2 * s0.numel() * 4)  # q, k, v, gate in; y out
    gbs = by / (ms / 1e3) / 1e9
    return {"steps": steps, "ms_per_step": round(ms, 4), "two_calls_ms_per_step": round(ms2, 4),
            "speedup_vs_two_calls": round(ms2 / ms, 3), "per": "head (dim channels)",
            "tokens_per_s": round(world * w.batch * w.seq / (ms / 1e3), 1), "algorithmic_bytes": by,
            "roofline": roofline("hbm", gbs, load_peaks()["hbm_gbs"], "GB/s",
                                 measured_traffic(w.name, "prefill_norm_gate"))}


GQA_BATCH, GQA_HEADS, GQA_KV_HEADS, GQA_CAP = 8, 64, 8, 131072


def run_gqa_leg(dev, stream, args, world):
    """lightning_gqa_decode: 8 sequences at the last position of a 131072-token
    bf16 cache, 64 query heads over 8 KV heads, RoPE on 64 dims; timed like the
    main leg. The step reads each sequence's whole cache once."""
    import torch
    import linear_attention_lightning_b200 as la
    from linear_attention_lightning_b200 import abi
    b, h, hk, cap, d = GQA_BATCH, GQA_HEADS, GQA_KV_HEADS, args.gqa_context, 128
    g = torch.Generator(device=dev).manual_seed(3000)
    mk = lambda *shape: torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    q, kn, vn = mk(b, h, d), mk(b, hk, d), mk(b, hk, d)
    kc, vc = mk(b, hk, cap, d), mk(b, hk, cap, d)
    pos = torch.full((b,), cap - 1, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    need = abi.lightning_gqa_decode_workspace_size(b, h, cap)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_gqa_decode(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                           abi.LA_DTYPE_BF16, pos.data_ptr(), b, h, hk, d, cap, 64, 1e4,
                                           1.0 / d ** 0.5, o.data_ptr(), ws.data_ptr(), need, sp))

    steps = args.gqa_steps
    ms = timed("gqa_decode", step, steps, args.warmup, stream, world, dev)
    # algorithmic bytes: the cache read for positions 0..cap-1 (K and V), the new k, v
    # written, q read and o written
    by = 2 * b * hk * cap * d * 2 + 2 * b * hk * d * 2 + 2 * b * h * d * 2
    gbs = by / (ms / 1e3) / 1e9
    return {"config": {"batch": b, "heads": h, "kv_heads": hk, "context": cap, "dim": d, "rot": 64,
                       "dtype": "bf16"},
            "steps": steps, "us_per_step": round(ms * 1e3, 2), "launches_per_step": 3,
            "roofline": roofline("hbm", gbs, load_peaks()["hbm_gbs"], "GB/s",
                                 measured_traffic("gqa_%d" % cap, "gqa_partial")),
            "l2": "cache %.1f GB per step > L2" % (by / 1e9)}


def run_gqa_prefill_leg(dev, stream, args, world):
    """lightning_gqa_prefill: one sequence of args.gqa_prefill_seq new tokens
    (empty cache), 64 query heads over 8 KV heads, RoPE on 64 dims, bf16;
    timed like the main leg. Causal FLOPs: 4 d per (query, key <= query) pair
    and query head (Q K^T and P V)."""
    import torch
    from linear_attention_lightning_b200 import abi
    b, h, hk, L, d = 1, GQA_HEADS, GQA_KV_HEADS, args.gqa_prefill_seq, 128
    g = torch.Generator(device=dev).manual_seed(3100)
    mk = lambda *shape: torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    q, kn, vn = mk(b, h, L, d), mk(b, hk, L, d), mk(b, hk, L, d)
    kc = torch.empty((b, hk, L, d), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    o = torch.empty_like(q)
    need = abi.lightning_gqa_prefill_workspace_size(abi.LA_DTYPE_BF16, b, h, L, d)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    start = torch.zeros((b,), dtype=torch.int32, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_gqa_prefill(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                            abi.LA_DTYPE_BF16, start.data_ptr(), b, h, hk, L, d, L, 64, 1e4,
                                            1.0 / d ** 0.5, o.data_ptr(), ws.data_ptr(), need, sp))

    steps = args.gqa_prefill_steps
    ms = timed("gqa_prefill", step, steps, args.warmup, stream, world, dev)
    peaks = load_peaks()
    causal = 4.0 * d * h * b * L * (L + 1) / 2
    tf = causal / (ms / 1e3) / 1e12
    # a timed region of several tenths of a second runs under the power cap
    peak, kind = tensor_peak(peaks, steps * ms / 1e3)
    rl = roofline("tensor", tf, peak, "TFLOP/s")
    rl["peak_kind"] = kind
    rl["frac_of_burst"] = round(tf / peaks["bf16_tflops"], 4)
    return {"config": {"batch": b, "heads": h, "kv_heads": hk, "seq": L, "dim": d, "rot": 64, "dtype": "bf16"},
            "steps": steps, "ms_per_step": round(ms, 3), "launches_per_step": 2,
            "tokens_per_s": round(world * b * L / (ms / 1e3), 1),
            "tflops_causal": round(tf, 2),
            "roofline": rl,
            "dram_bytes_per_launch": measured_traffic("gqa_prefill_%d" % L, "gqp_attn"),
            "flops": "causal: 4 d per (query, key <= query) pair and query head; the step includes the RoPE launch"}


def run_hybrid_leg(w, dev, stream, inp, vcode, dcode, args, world):
    """One block of the hybrid model's attention at the workload's shape: seven
    Lightning layers (prefill, then normalisation and gating of its output) and
    one softmax GQA layer (64 query heads over 8 KV heads, RoPE on 64 dims) on
    the same tokens, through the library's entry points; timed like the main
    leg. The layers reuse one set of inputs (timing only)."""
    import torch
    from linear_attention_lightning_b200 import abi
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    b, L, d = w.batch, w.seq, w.dim
    o = torch.empty_like(q)
    s_out = torch.empty((b, w.heads, d, d), dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev).manual_seed(w.seed + 4000)
    gate = torch.randn((b, L, w.heads * d), generator=g, device=dev).to(q.dtype)
    gamma = torch.ones(w.heads * d, device=dev)
    y = torch.empty((b, L, w.heads * d), dtype=q.dtype, device=dev)
    hq, hk = GQA_HEADS, GQA_KV_HEADS
    kn = torch.randn((b, hk, L, d), generator=g, device=dev).to(q.dtype)
    vn = torch.randn((b, hk, L, d), generator=g, device=dev).to(q.dtype)
    kc, vc = torch.empty_like(kn), torch.empty_like(vn)
    og = torch.empty((b, hq, L, d), dtype=q.dtype, device=dev)
    need = abi.lightning_gqa_prefill_workspace_size(dcode, b, hq, L, d)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    lneed = abi.lightning_prefill_workspace_size(b, w.heads, L, d, w.block)
    lws = torch.empty(max(lneed, 16), dtype=torch.uint8, device=dev)
    gstart = torch.zeros((b,), dtype=torch.int32, device=dev)
    sp = stream.cuda_stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def step(mark=False):
        if mark:
            ev[0].record(stream)
        for _ in range(7):
            abi.check(abi.lightning_prefill_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), dcode, sl.data_ptr(), b,
                                               w.heads, L, d, w.block, None if s0 is None else s0.data_ptr(),
                                               o.data_ptr(), s_out.data_ptr(), lws.data_ptr(), lneed, sp, vcode))
            abi.check(abi.lightning_norm_gate(o.data_ptr(), gate.data_ptr(), dcode, gamma.data_ptr(), 1e-6, b,
                                              w.heads, L, d, 0, y.data_ptr(), sp))
        if mark:
            ev[1].record(stream)
        abi.check(abi.lightning_gqa_prefill(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                            dcode, gstart.data_ptr(), b, hq, hk, L, d, L, 64, 1e4, 1.0 / d ** 0.5,
                                            og.data_ptr(), ws.data_ptr(), need, sp))
        if mark:
            ev[2].record(stream)

    for _ in range(max(1, min(args.warmup, 2))):
        step()
    steps = args.hybrid_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(steps):
        step(mark=(i == steps - 1))
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    check_device_status("hybrid_block", abi, sp, world, dev)
    lightning_ms, softmax_ms = ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])
    return {"layers": "7 x (Lightning prefill + norm and gate) + 1 x softmax GQA prefill", "steps": steps,
            "ms_per_step": round(ms, 3), "tokens_per_s": round(world * b * L / (ms / 1e3), 1),
            "lightning_ms": round(lightning_ms, 3), "softmax_ms": round(softmax_ms, 3),
            "softmax_share": round(softmax_ms / (lightning_ms + softmax_ms), 4)}


def run_hybrid_decode_leg(dev, stream, args, world):
    """One decode step of the hybrid block for GQA_BATCH sequences at a context of
    args.gqa_context tokens: seven Lightning decode steps (64 heads x 128, fp32
    states) and one softmax GQA decode step (64 query heads over 8 KV heads,
    bf16 cache), through the library's entry points."""
    import torch
    from linear_attention_lightning_b200 import abi, inputs
    b, h, hk, cap, d = GQA_BATCH, GQA_HEADS, GQA_KV_HEADS, args.gqa_context, 128
    g = torch.Generator(device=dev).manual_seed(3200)
    mk = lambda *shape: torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    states = [torch.randn((b, h, d, d), generator=g, device=dev) * 0.1 for _ in range(7)]
    sl = inputs.slopes(h, device=dev)
    ql, kl, vl = mk(b, h, d), mk(b, h, d), mk(b, h, d)
    ol = torch.empty_like(ql)
    q, kn, vn = mk(b, h, d), mk(b, hk, d), mk(b, hk, d)
    kc, vc = mk(b, hk, cap, d), mk(b, hk, cap, d)
    pos = torch.full((b,), cap - 1, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    need = abi.lightning_gqa_decode_workspace_size(b, h, cap)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    sp = stream.cuda_stream

    def step():
        for st in states:
            abi.check(abi.lightning_decode(ql.data_ptr(), kl.data_ptr(), vl.data_ptr(), abi.LA_DTYPE_BF16, sl.data_ptr(),
                                           b, h, d, st.data_ptr(), ol.data_ptr(), sp))
        abi.check(abi.lightning_gqa_decode(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                           abi.LA_DTYPE_BF16, pos.data_ptr(), b, h, hk, d, cap, 64, 1e4,
                                           1.0 / d ** 0.5, o.data_ptr(), ws.data_ptr(), need, sp))

    steps = args.gqa_steps
    ms = timed("hybrid_decode", step, steps, args.warmup, stream, world, dev)
    return {"layers": "7 x Lightning decode + 1 x softmax GQA decode", "sequences": b, "context": cap,
            "steps": steps, "us_per_step": round(ms * 1e3, 2), "tokens_per_s": round(world * b / (ms / 1e3), 1)}


def run_workload_leg(name, dev, stream, peaks, args, world):
    """The prefill on another named workload (the batched one with carried-in
    states: 16 sequences x 64 heads x 4096 tokens; the 8192-token one), timed
    like the main leg."""
    import torch
    import linear_attention_lightning_b200 as la
    from linear_attention_lightning_b200 import abi, inputs
    bw = inputs.WORKLOADS[name]
    inp = inputs.workload_inputs(bw, dev)
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    o = torch.empty_like(q)
    s_out = torch.empty((bw.batch, bw.heads, bw.dim, bw.dim), dtype=torch.float32, device=dev)
    variant = la.prefill_variant(bw.dtype, bw.batch, bw.heads, bw.seq, bw.dim, bw.block)
    vcode = {"simt": abi.LA_VARIANT_SIMT, "tcgen05": abi.LA_VARIANT_TCGEN05,
             "pair": abi.LA_VARIANT_TCGEN05_PAIR}[variant]
    need = abi.lightning_prefill_workspace_size(bw.batch, bw.heads, bw.seq, bw.dim, bw.block)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_prefill_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), abi.LA_DTYPE_BF16, sl.data_ptr(),
                                           bw.batch, bw.heads, bw.seq, bw.dim, bw.block,
                                           None if s0 is None else s0.data_ptr(), o.data_ptr(), s_out.data_ptr(),
                                           ws.data_ptr(), need, sp, vcode))

    steps = args.batched_steps
    ms = timed("other_workloads/%s" % bw.name, step, steps, args.warmup, stream, world, dev)
    by = prefill_bytes(bw.batch, bw.heads, bw.seq, bw.dim, 2, state_in=s0 is not None, state_out=True)
    gbs = by / (ms / 1e3) / 1e9
    fl = prefill_flops(bw.batch, bw.heads, bw.seq, bw.dim, bw.block)["formula"] / (ms / 1e3) / 1e12
    return {"workload": bw.name, "kernel": variant, "steps": steps, "ms_per_step": round(ms, 4),
            "tokens_per_s": round(world * bw.batch * bw.seq / (ms / 1e3), 1), "tflops_formula": round(fl, 2),
            "roofline": roofline("hbm", gbs, peaks["hbm_gbs"], "GB/s", measured_traffic(bw.name, variant))}


def run_backward_leg(w, dev, stream, inp, dcode, args, world):
    """lightning_prefill_backward on the workload (AUTO: the CTA-pair tensor-core
    kernel where it applies), timed like the main leg: dQ causal on (dO, V, K),
    dV and dK anti-causal on (K, Q, dO) and (V, dO, Q)."""
    import torch
    from linear_attention_lightning_b200 import abi
    q, k, v, sl, s0 = inp["q"], inp["k"], inp["v"], inp["slopes"], inp["state_in"]
    g = torch.Generator(device=dev).manual_seed(w.seed + 1000)
    d_o = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
    d_so = torch.randn((w.batch, w.heads, w.dim, w.dim), generator=g, device=dev) * 0.1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ds_in = torch.empty_like(d_so)
    variant = abi.LA_VARIANT_AUTO
    need = abi.lightning_prefill_backward_workspace_size(dcode, w.batch, w.heads, w.seq, w.dim, w.block, variant)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sp = stream.cuda_stream

    def step():
        abi.check(abi.lightning_prefill_backward(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), d_o.data_ptr(), dcode, sl.data_ptr(), w.batch, w.heads,
            w.seq, w.dim, w.block, None if s0 is None else s0.data_ptr(), d_so.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), ds_in.data_ptr(), ws.data_ptr(), need, sp, variant))

    steps = args.backward_steps
    ms = timed("backward", step, steps, args.warmup, stream, world, dev)
    peaks = load_peaks()
    eb = 2 if q.dtype == torch.bfloat16 else 4
    # algorithmic bytes: q, k, v, dO read and dq, dk, dv written once, plus the
    # fp32 states (state_in, d_state_out read, d_state_in written)
    units = w.batch * w.heads * w.seq
    by = 7 * units * w.dim * eb + 3 * w.batch * w.heads * w.dim * w.dim * 4
    gbs = by / (ms / 1e3) / 1e9
    # three passes of the block recurrence: 3 x (4Bd + 4d^2) per (token, head)
    tf = 3 * prefill_flops(w.batch, w.heads, w.seq, w.dim, w.block)["formula"] / (ms / 1e3) / 1e12
    import linear_attention_lightning_b200 as la
    try:
        la.prefill_variant(w.dtype, w.batch, w.heads, w.seq, w.dim, w.block, "pair")
        kernel = "pair (dQ causal, dV and dK anti-causal)"
    except ValueError:
        kernel = "simt (3 passes)"
    return {"kernel": kernel, "steps": steps, "ms_per_step": round(ms, 3),
            "tokens_per_s": round(world * w.batch * w.seq / (ms / 1e3), 1),
            "workspace_bytes": need,
            "roofline": roofline("hbm", gbs, peaks["hbm_gbs"], "GB/s",
                                 measured_traffic(w.name, "backward_pair", "dram_bytes_per_step")),
            "tflops_formula": round(tf, 2),
            "frac_bf16_peak_formula": round(tf / peaks["bf16_tflops"], 4)}


def abi_ws_bytes(w):
    from linear_attention_lightning_b200 import abi
    return abi.lightning_prefill_workspace_size(w.batch, w.heads, w.seq, w.dim, w.block)


def run_e2e(w, dev, stream, inp, variant, args, world):
    """Same prefill through the public API with host buffers: every step copies
    q, k, v from pinned host memory and reads o and the state back. Steps are
    pipelined over two device buffer sets: step i's inputs copy in on one
    stream while step i-1 computes and its outputs copy out on another (the
    two PCIe directions have their own copy engines)."""
    import torch
    import linear_attention_lightning_b200 as la
    steps = args.e2e_steps
    hq = inp["q"].cpu().pin_memory()
    hk = inp["k"].cpu().pin_memory()
    hv = inp["v"].cpu().pin_memory()
    ho = torch.empty_like(hq).pin_memory()
    hs = torch.empty((w.batch, w.heads, w.dim, w.dim), dtype=torch.float32).pin_memory()
    sets = [[torch.empty_like(inp["q"]) for _ in range(3)] for _ in range(2)]
    outs = [(torch.empty_like(inp["q"]), torch.empty((w.batch, w.heads, w.dim, w.dim), dtype=torch.float32,
                                                      device=dev)) for _ in range(2)]
    wsp = torch.empty(max(abi_ws_bytes(w), 16), dtype=torch.uint8, device=dev)
    h2d = 3 * hq.numel() * hq.element_size()
    d2h = ho.numel() * ho.element_size() + hs.numel() * 4
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()

    def run(n):
        copied = [None, None]  # per buffer set: inputs landed
        computed = [None, None]  # per buffer set: compute done (inputs free, outputs ready)
        read = [None, None]      # per buffer set: outputs copied out
        for i in range(n):
            b = i % 2
            dq, dk, dv = sets[b]
            o, s_ = outs[b]
            with torch.cuda.stream(s_in):
                if computed[b] is not None:
                    s_in.wait_event(computed[b])   # the compute two steps back read this set
                dq.copy_(hq, non_blocking=True)
                dk.copy_(hk, non_blocking=True)
                dv.copy_(hv, non_blocking=True)
                copied[b] = ev()
                copied[b].record(s_in)
            stream.wait_event(copied[b])
            if read[b] is not None:
                stream.wait_event(read[b])         # its outputs from two steps back were read
            la.prefill(dq, dk, dv, inp["slopes"], w.block, inp["state_in"], variant=variant, o=o, state_out=s_,
                       workspace=wsp, stream=stream)
            computed[b] = ev()
            computed[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                ho.copy_(o, non_blocking=True)
                hs.copy_(s_, non_blocking=True)
                read[b] = ev()
                read[b].record(s_out)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)

    run(1)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    from linear_attention_lightning_b200 import abi
    check_device_status("e2e", abi, stream.cuda_stream, world, dev)
    value = world * w.batch * w.seq * steps / (ms / 1e3)
    # the last step's host output is the device prefill's on the same inputs
    ref_o, _ = la.prefill(inp["q"], inp["k"], inp["v"], inp["slopes"], w.block, inp["state_in"], variant=variant)
    same = bool(torch.equal(ho, ref_o.cpu()))
    return {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "output_matches_device_call": same,
            "pipeline": "two buffer sets; inputs in on one stream, outputs out on another"}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=PREFILL_WORKLOAD)
    p.add_argument("--decode-steps", type=int, default=1000)
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--gqa-steps", type=int, default=20,
                   help="timed steps of the softmax GQA decode leg (0 skips it)")
    p.add_argument("--gqa-context", type=int, default=GQA_CAP,
                   help="cached tokens per sequence in the GQA decode leg")
    p.add_argument("--gqa-prefill-steps", type=int, default=3,
                   help="timed steps of the softmax GQA prefill leg (0 skips it)")
    p.add_argument("--gqa-prefill-seq", type=int, default=131072,
                   help="new tokens of the GQA prefill leg")
    p.add_argument("--batched-steps", type=int, default=5,
                   help="timed steps of the other prefill workloads' legs (0 skips them)")
    p.add_argument("--hybrid-steps", type=int, default=2,
                   help="timed steps of the hybrid-block leg, 7 Lightning + 1 softmax layer (0 skips it)")
    p.add_argument("--norm-gate-steps", type=int, default=20,
                   help="timed steps of the norm-and-gate epilogue leg (0 skips it)")
    p.add_argument("--fused-norm-gate-steps", type=int, default=10,
                   help="timed steps of the prefill with the per-head norm + gate fused in (0: skip)")
    p.add_argument("--backward-steps", type=int, default=10,
                   help="timed steps of the gradient leg (0 skips it)")
    p.add_argument("--variant", choices=["auto", "pair", "tcgen05", "simt"], default="auto",
                   help="prefill kernel of the main leg (auto: the library's choice for the workload)")
    p.add_argument("--block", type=int, default=0,
                   help="block length of the main leg (0: the workload's own)")
    p.add_argument("--snapshot-interval", type=int, default=16384,
                   help="tokens between prefix-cache state snapshots in the snapshot leg (0 skips it)")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be at least 3")
    if a.gqa_context < 1:
        p.error("--gqa-context must be positive")
    return a


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
