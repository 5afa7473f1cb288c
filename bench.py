#!/usr/bin/env python
"""Benchmark of the jagged-attention hot path (libjfa) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {jfa,reference}]
                    [--workload self_bf16]

One step = the whole path over one synthetic batch held in HBM: schedule +
forward (scores, bias, mask, online softmax or GDPA activation, P.V, LSE) +
backward (D = rowsum(dO*O), dQ, dK, dV), all through the C ABI.  The metric is
TFLOP/s counted on valid (unpadded) query/key pairs only: forward 4*d per pair
and head, backward 2.5x that (five GEMMs including the score recompute);
softmax/exp/bias work is not counted.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronisation, timed with CUDA events on the launching stream; the
max over ranks is reported.  Every input tensor of the default workload is
larger than L2 (126 MB), so no L2 flush is needed between steps.  Under
torchrun (N ranks) the job is one global batch of N x B sequences of the
workload: every rank draws the same global lengths, splits them with
jfa_partition (base batch shuffling by default, or LPT), and draws and runs
only its own sequences -- weak scaling, no collective on the data path.  The
line reports the split's rank imbalance (heaviest rank's visible pairs over
the mean) beside that of a plain contiguous split.

Also reported on one JSON line: per-kernel launch times from the library's
event hooks (the dominant kernel's roofline fraction), the end-to-end number
through the C ABI with host buffers (pinned host -> device copies of the
inputs and device -> host copies of every result inside the timed region),
a padded-dense baseline (torch SDPA on the max-padded batch, causal, no
bias), the CPU oracle on a bounded sample of the same batch, and the SM
clocks sampled during the timed region.

``--impl reference`` times the fp64 CPU oracle (the only other implementation
of this method) on the host cores, each step a bounded stratified sample of
the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "jagged attn fwd/bwd TFLOP/s (valid tokens); % of B200 dense BF16/FP8 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SM_COUNT = 148
FP32_LANES_PER_SM = 128


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["jfa", "reference"], default="jfa")
    ap.add_argument("--workload", default="self_bf16")
    ap.add_argument("--act", default=None, help="override the workload's activation")
    ap.add_argument("--bias", default=None, choices=["none", "relpos", "dense"],
                    help="override the workload's bias kind (a what-if: the metric's workload keeps its own)")
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's number of sequences (profiling captures)")
    ap.add_argument("--max-len", type=int, default=None,
                    help="override the workload's length clip (profiling captures)")
    ap.add_argument("--block", type=int, default=0,
                    help="BlockAttention block length (self-attention workloads); 0 = full")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding-window width (query at position p sees keys p - w < j); 0 = none")
    ap.add_argument("--partition", choices=["bbs", "lpt"], default="bbs",
                    help="split of the global batch across ranks (N > 1)")
    ap.add_argument("--sub-batch", type=int, default=8,
                    help="sequences per sub-batch for --partition bbs")
    ap.add_argument("--e2e-steps", type=int, default=16,
                    help="timed steps of the end-to-end leg (its pipeline fills and drains once)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-padded", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mx-internal", action="store_true",
                    help="MXFP8: run jfa_forward / jfa_backward with dtype MXFP8 (quantising inside "
                         "each call) instead of the producer form of the step")
    ap.add_argument("--copy-probe", action="store_true",
                    help="time pinned host<->device copies of the e2e leg's size (in alone, out "
                         "alone, both at once on two streams), print one JSON line and exit")
    ap.add_argument("--fp8-peak-probe", action="store_true",
                    help="time the library FP8 GEMM (E4M3, and MX-scaled where supported) at 8192^3 "
                         "as the fp8 roofline denominator, print one JSON line and exit")
    ap.add_argument("--cpu-sample-pairs", type=float, default=8e6,
                    help="(query, key) pairs x heads in the CPU oracle's sample")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# work accounting
# ---------------------------------------------------------------------------
def visible_pairs(q_lens, kv_lens, causal, block=0, window=0):
    """Per-sequence number of (query, key) pairs attention computes; with
    BlockAttention (block > 0, self-attention) only pairs inside a block, with
    a sliding window (window > 0) only pairs with p - j < window (and, without
    the causal rule, j - p < window), p = i + n_kv - n_q."""
    out = np.zeros(len(q_lens), np.int64)
    for b, (nq, nk) in enumerate(zip(q_lens, kv_lens)):
        nq, nk = int(nq), int(nk)
        if block > 0:
            m = np.minimum(block, nq - np.arange(0, nq, block)).astype(np.int64)
            out[b] = int((m * (m + 1) // 2).sum() if causal else (m * m).sum())
        elif window > 0:
            pos = np.arange(nq, dtype=np.int64) + nk - nq
            hi = np.minimum(nk - 1, pos if causal else pos + window - 1)
            lo = np.maximum(0, pos - window + 1)
            out[b] = int(np.maximum(hi - lo + 1, 0).sum())
        elif not causal:
            out[b] = nq * nk
        else:
            i = np.arange(nq, dtype=np.int64)
            out[b] = int(np.clip(i + 1 + nk - nq, 0, nk).sum())
    return out


def sq_bytes(p, backward: bool, softmax: bool) -> float:
    """Algorithmic HBM bytes of one short-query kernel launch: every operand
    read once and every result written once.  Forward: Q, K, V, the dense
    bias, O (and the fp32 LSE).  Backward: Q, K, V, dO, the dense bias, LSE
    and D (fp32), written dQ, dK, dV."""
    el = 2 if p.dtype != "f32" else 4
    tq = float(p.total_q) * p.H * p.d * el
    tkv = float(p.kv_off[-1]) * p.H * p.d * el
    bias = float(p.bias.numel()) * el if p.bias_kind == "dense" else 0.0
    rows = float(p.total_q) * p.H * 4
    if not backward:
        return tq + 2 * tkv + bias + tq + (rows if softmax else 0.0)
    return 2 * tq + 2 * tkv + bias + (2 * rows if softmax else 0.0) + tq + 2 * tkv


def flops_of(p, pairs_per_seq=None, block=0, window=0):
    pairs = (visible_pairs(p.q_lens, p.kv_lens, p.causal, block, window) if pairs_per_seq is None
             else pairs_per_seq)
    f_fwd = 4.0 * p.d * p.H * float(pairs.sum())
    return f_fwd, 2.5 * f_fwd


def padded_flops(p):
    L = int(max(p.max_q_len, p.max_kv_len))
    per = L * (L + 1) // 2 if p.causal else L * L
    f_fwd = 4.0 * p.d * p.H * p.B * per
    return f_fwd, 2.5 * f_fwd


# ---------------------------------------------------------------------------
# peaks, clocks, profiles
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML (read-only queries)
    every 5 ms on a host thread, so that a timed region of a few tens of
    milliseconds still gets samples."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                mask = get_reasons(self.handle) if get_reasons else 0
                self.samples.append((sm, mask))
            except Exception:
                pass
            self.stop_evt.wait(0.005)

    def start(self):
        self.thread.start()

    def stop(self):
        self.stop_evt.set()
        self.thread.join(timeout=2)
        nv = self.nv
        try:
            smax = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
        except Exception:
            smax = None
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"], "source": "nvml"}
        reasons = sorted({name for _, m in self.samples for name, attr in self.REASONS
                          if hasattr(nv, attr) and (m & getattr(nv, attr))})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def clock_sampler(device_index):
    """NVML sampler when the binding is there, else nvidia-smi."""
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons (every 200 ms)."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(", ") for r in self.tmp.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        mine = [r for r in rows if len(r) >= 10 and (self.uuid is None or r[1] == self.uuid)]
        if not mine:
            mine = [r for r in rows if len(r) >= 10 and r[0] == "0"]
        if not mine:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in mine if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in mine if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in mine for k in range(4) if r[6 + k].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(mine)}


def kernel_source_hash(name):
    src = {"tc_fwd": "jfa_tc_fwd.cu", "tc_bwd": "jfa_tc_bwd.cu", "tc_fwd_sq": "jfa_tc_fwd_sq.cu",
           "tc_bwd_sq": "jfa_tc_bwd_sq.cu", "tc_fwd_mxfp8": "jfa_tc_fwd_mx.cu", "simt_fwd": "jfa_simt.cu",
           "simt_bwd_dq": "jfa_simt.cu", "simt_bwd_dkdv": "jfa_simt.cu"}.get(name)
    if src is None:
        return None
    path = os.path.join(ROOT, "jagged_attention_recommender_jfa_b200", "csrc", src)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256") != kernel_source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_full_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# reference arm / CPU baseline: the fp64 oracle on a bounded stratified sample
# ---------------------------------------------------------------------------
def cpu_sample_mask(p, target_pairs_heads, block=0, window=0):
    """Sequences picked evenly over the length-sorted batch (shortest first)
    until the sample holds ~target (pairs x heads)."""
    pairs = visible_pairs(p.q_lens, p.kv_lens, p.causal, block, window) * p.H
    order = np.argsort(pairs, kind="stable")
    mask = np.zeros(p.B, np.int32)
    total = 0
    for stride in (64, 32, 16, 8, 4, 2, 1):
        for idx in order[::stride]:
            if mask[idx]:
                continue
            if total + pairs[idx] > target_pairs_heads and total > 0:
                continue
            mask[idx] = 1
            total += int(pairs[idx])
        if total >= 0.5 * target_pairs_heads:
            break
    return mask, pairs


def run_oracle_step(p, mask, act, block=0, window=0):
    import oracle
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
              causal=p.causal, seq_mask=mask, block=block, window=window)
    o, l = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw)


def cpu_baseline(p, act, target, block=0, window=0):
    import oracle
    mask, pairs = cpu_sample_mask(p, target, block, window)
    f_fwd = 4.0 * p.d * float((pairs * mask).sum())
    t0 = time.perf_counter()
    run_oracle_step(p, mask, act, block, window)
    dt = time.perf_counter() - t0
    n = int(mask.sum())
    return {"value": 3.5 * f_fwd / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{n} of {p.B} sequences (all {p.H} heads, stratified by length), "
                      f"{int((pairs * mask).sum())} pair-heads, fwd+bwd fp64, {dt:.1f} s"}


def reference_arm(args, rank, world):
    if rank != 0:
        return
    from jagged_attention_recommender_jfa_b200.inputs import make_problem
    import oracle
    p = make_problem(args.workload, args.seed, B=args.batch, max_len=args.max_len, bias=args.bias)
    act = args.act or p.act
    target = args.cpu_sample_pairs / 4
    mask, pairs = cpu_sample_mask(p, target, args.block, args.window)
    f_sample = 3.5 * 4.0 * p.d * float((pairs * mask).sum())
    for _ in range(args.warmup):
        run_oracle_step(p, mask, act, args.block, args.window)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_step(p, mask, act, args.block, args.window)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = f_sample / dt / 1e12
    n = int(mask.sum())
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "global_batch": p.B, "heads": p.H,
                   "head_dim": p.d, "act": act, "causal": p.causal, "block": args.block or None,
                   "window": args.window or None, "sample_sequences": n, "l2": "inputs larger than L2"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"each step: {n} of {p.B} sequences (stratified by length), "
                                   f"all heads, fwd+bwd fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# padded-dense baseline: torch SDPA on the max-padded batch
# ---------------------------------------------------------------------------
def padded_dense_baseline(p, dev, f_valid, iters=3):
    L = int(max(p.max_q_len, p.max_kv_len))
    need = 10 * p.B * p.H * L * p.d * 2
    free, _ = torch.cuda.mem_get_info(dev)
    if need > 0.6 * free:
        return {"skipped": f"needs {need / 1e9:.1f} GB"}
    import torch.nn.functional as F
    try:
        q = torch.randn(p.B, p.H, L, p.d, device=dev, dtype=torch.bfloat16, requires_grad=True)
        k = torch.randn_like(q, requires_grad=True)
        v = torch.randn_like(q, requires_grad=True)
        go = torch.randn_like(q)

        def once():
            o = F.scaled_dot_product_attention(q, k, v, is_causal=p.causal)
            o.backward(go)

        once()
        torch.cuda.synchronize(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(iters):
            once()
        e.record()
        torch.cuda.synchronize(dev)
        ms = s.elapsed_time(e) / iters
        pf, pb = padded_flops(p)
        return {"impl": "torch SDPA (padded to max_len, causal, no bias)", "ms_per_step": ms,
                "valid_token_tflops": f_valid / (ms * 1e-3) / 1e12,
                "padded_tflops": (pf + pb) / (ms * 1e-3) / 1e12, "max_len": L}
    finally:
        for name in ("q", "k", "v", "go"):
            locals().pop(name, None)
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# main arm
# ---------------------------------------------------------------------------
def fp8_peak_probe(dev, n=8192, warmup=5, iters=20):
    """Dense FP8 tensor-core throughput of the library GEMM (cuBLASLt through
    torch._scaled_mm) at n^3, E4M3 x E4M3 -> bf16: with per-tensor scales, and
    with MX block scales (one E8M0 per 32 elements along K, all 2^0, so their
    layout does not matter) where this build supports them.  Timed with CUDA
    events after warm-up; the MXFP8 attention kernel's fp8 roofline."""
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)   # [N][K]: b.t() is K x N column-major
    one = torch.ones((), device=dev)

    def tflops(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(iters):
            fn()
        t1.record()
        torch.cuda.synchronize()
        return 2.0 * n ** 3 / (t0.elapsed_time(t1) / iters * 1e-3) / 1e12

    out = {"probe": "fp8_peak", "n": n, "iters": iters,
           "fp8_e4m3_tflops": tflops(lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one,
                                                              out_dtype=torch.bfloat16))}
    try:
        def rup(x, m):
            return (x + m - 1) // m * m
        ns = rup(n, 128) * rup(n // 32, 4)
        sa = torch.full((ns,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
        sb = torch.full((ns,), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
        out["mxfp8_tflops"] = tflops(lambda: torch._scaled_mm(a, b.t(), scale_a=sa, scale_b=sb,
                                                              out_dtype=torch.bfloat16))
    except Exception as e:   # noqa: BLE001 -- reported, not fatal
        out["mxfp8_tflops"] = None
        out["mxfp8_unavailable"] = str(e).splitlines()[0][:200]
    out["device"] = torch.cuda.get_device_name(dev)
    return out


def copy_probe(dev, nbytes=1_821_206_568, reps=5):
    """Host link bandwidth for the end-to-end leg: pinned host memory to the
    device, back, and both directions at once on two streams, timed with
    CUDA events; nbytes is one self_bf16 step's input (Q, K, V, dO, offsets,
    bias table)."""
    h_in = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    h_out = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_out = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def timed(do_in, do_out):
        ms = []
        for _ in range(reps + 1):
            torch.cuda.synchronize(dev)
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            up.wait_event(t0)
            down.wait_event(t0)
            if do_in:
                with torch.cuda.stream(up):
                    d_in.copy_(h_in, non_blocking=True)
            if do_out:
                with torch.cuda.stream(down):
                    h_out.copy_(d_out, non_blocking=True)
            cur = torch.cuda.current_stream(dev)
            cur.wait_stream(up)
            cur.wait_stream(down)
            t1.record()
            torch.cuda.synchronize(dev)
            ms.append(t0.elapsed_time(t1))
        return statistics.median(ms[1:])

    res = {"probe": "host_copies", "bytes_per_direction": nbytes}
    for name, a, b in (("h2d", True, False), ("d2h", False, True), ("both", True, True)):
        ms = timed(a, b)
        res[name + "_ms"] = ms
        res[name + "_gbs_per_direction"] = nbytes / (ms * 1e-3) / 1e9
    return res


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl jfa needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.fp8_peak_probe:
        if rank == 0:
            print(json.dumps(fp8_peak_probe(dev)))
        return
    if args.copy_probe:
        if rank == 0:
            print(json.dumps(copy_probe(dev)))
        return
    from jagged_attention_recommender_jfa_b200 import jfa
    from jagged_attention_recommender_jfa_b200.inputs import WORKLOADS, draw_lengths

    p, split = rank_problem(args, rank, world, jfa)
    act = args.act or p.act
    if args.block and args.window:
        raise SystemExit("--block and --window are alternatives")
    prob = jfa.problem_of(p, window=args.window)
    path = jfa.jfa_path(prob, act, 0), jfa.jfa_path(prob, act, 1)
    f_fwd, f_bwd = flops_of(p, block=args.block, window=args.window)
    d = {n: getattr(p, n).to(dev).contiguous() for n in ("q", "k", "v", "dout", "q_off", "kv_off")}
    seq_off = d["q_off"]
    if args.block:
        # BlockAttention: the same kernels over the blocks; the offsets are
        # rewritten inside every timed step
        if not torch.equal(p.q_off, p.kv_off):
            raise SystemExit("--block needs a self-attention workload")
        prob, boff = jfa.block_attention(prob, seq_off, args.block)
        d["q_off"] = d["kv_off"] = boff
    bias = p.bias.to(dev).contiguous() if p.bias is not None else None
    out = torch.empty_like(d["q"])
    lse = torch.empty(p.total_q, p.H, dtype=torch.float32, device=dev) if act == "softmax" else None
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    apass = AttentionPass(jfa, prob, p, act, dev, internal=args.mx_internal)
    ws_f, ws_b = apass.workspaces
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(marks=None):
        if marks is not None:
            marks[0].record(stream)
        if args.block:
            jfa.jfa_block_offsets(seq_off, p.B, p.total_q, args.block, d["q_off"], stream=stream)
        apass.forward(d, d["q_off"], d["kv_off"], bias, out, lse, stream)
        if marks is not None:
            marks[1].record(stream)
        apass.backward(d, d["q_off"], d["kv_off"], bias, out, lse, dq, dk, dv, stream)
        if marks is not None:
            marks[2].record(stream)

    for _ in range(args.warmup):
        step()
    jfa.jfa_check_error(ws_f, stream)
    jfa.jfa_check_error(ws_b, stream)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = clock_sampler(local)
    clocks.start()
    if isinstance(clocks, ClockSampler):
        time.sleep(0.3)   # nvidia-smi needs a moment before its first sample
    marks = [[ev(), ev(), ev()] for _ in range(args.steps)]
    t_start, t_end = ev(), ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    jfa.jfa_profile_enable(True)
    t_start.record(stream)
    for k in range(args.steps):
        step(marks[k])
    t_end.record(stream)
    jfa.jfa_profile_enable(False)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    fwd_ms = sum(m[0].elapsed_time(m[1]) for m in marks) / args.steps
    bwd_ms = sum(m[1].elapsed_time(m[2]) for m in marks) / args.steps
    launches = jfa.jfa_profile_read()
    jfa.jfa_check_error(ws_f, stream)
    jfa.jfa_check_error(ws_b, stream)

    ms_step = ms_total / args.steps
    flops_rank = f_fwd + f_bwd
    ms_step_max, flops_all = aggregate_over_ranks(ms_step, flops_rank, dev, world)
    value = flops_all / (ms_step_max * 1e-3) / 1e12

    # per-kernel totals over the timed region
    per = {}
    for name, ms in launches:
        c = per.setdefault(name, [0, 0.0])
        c[0] += 1
        c[1] += ms
    dom = max(per.items(), key=lambda kv: kv[1][1])[0] if per else None
    peaks, peak_src = load_peaks()
    kernels = {n: {"launches": c, "total_ms": round(t, 4), "share": round(t / ms_total, 4)}
               for n, (c, t) in sorted(per.items(), key=lambda kv: -kv[1][1])}
    roofline = None
    if dom is not None:
        avg_s = per[dom][1] / per[dom][0] * 1e-3
        d_ = p.d
        pairs = f_fwd / (4.0 * d_)
        algo = {"tc_fwd": f_fwd, "tc_fwd_mxfp8": f_fwd, "tc_bwd": f_bwd, "simt_fwd": f_fwd,
                "simt_bwd_dq": 6.0 * d_ * pairs, "simt_bwd_dkdv": 8.0 * d_ * pairs}.get(dom)
        if dom in ("tc_fwd_sq", "tc_bwd_sq"):
            # short query sequences: the pair work is small against the bytes
            # every operand costs once, so HBM bounds these kernels
            algo = sq_bytes(p, dom == "tc_bwd_sq", act == "softmax")
            peak = peaks["hbm_gbs"]
            bound, unit = "hbm", "GB/s"
            note = f"HBM copy bandwidth of {peak_src}"
            achieved = algo / avg_s / 1e9
        elif dom == "tc_fwd_mxfp8":
            # E4M3 block-scaled MMAs: the measured bf16 peak x the nominal
            # fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense)
            peak = 2.0 * peaks["bf16_tflops"]
            bound, unit = "tensor", "TFLOP/s"
            note = f"fp8 dense = 2 x bf16 burst of {peak_src}"
        elif dom.startswith("tc_"):
            # the kernel runs for milliseconds inside a sub-second timed
            # region: the burst figure applies
            peak = peaks["bf16_tflops"]
            bound, unit = "tensor", "TFLOP/s"
            note = f"bf16 dense, burst, of {peak_src}"
        else:
            mhz = peaks.get("sm_max_mhz", 1965.0)
            peak = SM_COUNT * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
            bound, unit = "alu", "TFLOP/s"
            note = f"fp32 FMA: {SM_COUNT} SMs x {FP32_LANES_PER_SM} lanes x 2 x {mhz:.0f} MHz"
        if bound != "hbm":
            achieved = algo / avg_s / 1e12 if algo else None
        traffic = recorded_traffic(dom, args.workload)
        roofline = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
                    "unit": unit, "frac": achieved / peak if achieved else None,
                    "traffic": traffic, "peak_source": note,
                    ("algorithmic_bytes_per_launch" if bound == "hbm"
                     else "algorithmic_flops_per_launch"): algo,
                    "avg_launch_ms": avg_s * 1e3}

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if path[0] == 1 else "f32",
        "data": "synthetic",
        "config": {"workload": args.workload if args.batch is None and args.max_len is None
                   else f"{args.workload} (B={p.B}, max_len={args.max_len})",
                   "global_batch": (args.batch or WORKLOADS[args.workload]["B"]) * world,
                   "heads": p.H,
                   "head_dim": p.d, "act": act, "causal": p.causal, "bias": p.bias_kind,
                   "total_tokens": p.total_q, "max_len": p.max_q_len,
                   "block": args.block or None, "window": args.window or None,
                   "parallelism": (f"dp{world} ({args.partition} split of one global batch)"
                                   if world > 1 else "dp1"),
                   "l2": "inputs larger than L2 (each of Q/K/V/dO > 126 MB); no flush",
                   "kernel_path": {"fwd": "tcgen05" if path[0] == 1 else "cuda-core",
                                   "bwd": "tcgen05" if path[1] == 1 else "cuda-core"}},
        "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
        "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
        "pct_of_bf16_burst_peak": {"fwd": 100 * f_fwd / (fwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                   "bwd": 100 * f_bwd / (bwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]},
        # the MXFP8 forward against the fp8 peak (2 x the measured bf16 burst)
        "pct_of_fp8_burst_peak": ({"fwd": 50 * f_fwd / (fwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}
                                  if p.dtype == "mxfp8" else None),
        "roofline": roofline,
        "kernels": kernels,
        "gpu_launches": len(launches),
        "clocks": clock_info,
    }

    # rank balance of the split: this run's (N > 1), and what an 8-rank split
    # of 8 x B sequences of this workload would give (host-side only)
    if split is not None:
        result["partition"] = split
    else:
        gq, gk = draw_lengths(args.workload, args.seed, B=8 * p.B, max_len=args.max_len)
        result["partition_8_ranks"] = {
            m: split_report(gq, gk, p.causal, 8, m, args.sub_batch, jfa, args.window)[1] for m in ("bbs", "lpt")}

    # end to end through the C ABI with host buffers
    if not args.no_e2e:
        result["e2e"] = e2e_leg(args, p, prob, act, dev, stream, jfa, f_fwd + f_bwd, world)
    if rank == 0 and world == 1 and not args.no_padded and not args.block and not args.window:
        result["padded_dense_baseline"] = padded_dense_baseline(p, dev, f_fwd + f_bwd)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(p, act, args.cpu_sample_pairs, args.block,
                                              args.window)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def split_report(q_lens, kv_lens, causal, ranks, method, sub_batch, jfa, window=0):
    """Rank imbalance (heaviest rank's visible pairs / mean) of the chosen
    split and of a contiguous split (rank r takes the r-th run of B/N)."""
    rank_of, cost = jfa.jfa_partition(q_lens, kv_lens, causal, ranks, method, sub_batch, window)
    per = len(q_lens) // ranks
    contiguous = np.minimum(np.arange(len(q_lens)) // max(per, 1), ranks - 1).astype(np.int32)
    pairs = visible_pairs(q_lens, kv_lens, causal, 0, window)
    c_cost = np.bincount(contiguous, weights=pairs, minlength=ranks)
    imb = lambda c: float(np.max(c) / np.mean(c)) if np.mean(c) > 0 else 1.0
    return rank_of, {"method": method, "sub_batch": sub_batch if method == "bbs" else None,
                     "ranks": ranks, "sequences": int(len(q_lens)),
                     "imbalance_max_over_mean": imb(cost),
                     "contiguous_imbalance_max_over_mean": imb(c_cost)}


def rank_problem(args, rank, world, jfa):
    """This rank's batch.  One rank: the workload's batch (seed args.seed).
    N ranks: the global batch of N x B sequences (lengths from args.seed, the
    same on every rank), split by jfa_partition; this rank draws the tensors
    of its own sequences only (seed args.seed + 1 + rank)."""
    from jagged_attention_recommender_jfa_b200.inputs import WORKLOADS, draw_lengths, make_problem
    if world == 1:
        return make_problem(args.workload, args.seed, B=args.batch, max_len=args.max_len, bias=args.bias), None
    B = args.batch or WORKLOADS[args.workload]["B"]
    q_lens, kv_lens = draw_lengths(args.workload, args.seed, B=B * world, max_len=args.max_len)
    causal = WORKLOADS[args.workload]["causal"]
    rank_of, report = split_report(q_lens, kv_lens, causal, world, args.partition,
                                   args.sub_batch, jfa, args.window)
    mine = np.nonzero(rank_of == rank)[0]
    p = make_problem(args.workload, args.seed + 1 + rank, q_lens=q_lens[mine],
                     kv_lens=kv_lens[mine], max_len=args.max_len, bias=args.bias)
    return p, report


def aggregate_over_ranks(ms_per_step, flops, device, world):
    """Whole-job numbers of one timed region: the slowest rank's time per step
    and the work of all ranks (weak scaling: every rank runs its own batch).
    Returns (max ms per step, summed flops)."""
    if world <= 1:
        return float(ms_per_step), float(flops)
    import torch.distributed as dist
    t = torch.tensor([ms_per_step], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    fl = torch.tensor([flops], dtype=torch.float64, device=device)
    dist.all_reduce(fl, op=dist.ReduceOp.SUM)
    return float(t.item()), float(fl.item())


class AttentionPass:
    """One forward + backward of the library on device inputs.  MXFP8 runs in
    its producer form: one quantisation pass per operand writes the E4M3 codes
    for jfa_forward_mxfp8 and the dequantised operands for a bf16
    jfa_backward, which is then the MXFP8 backward (bf16 gradients on the
    values the forward's block-scaled MMAs saw), so nothing is quantised
    twice; ``internal`` runs jfa_forward / jfa_backward with dtype MXFP8
    instead, which quantise inside the call."""

    def __init__(self, jfa, prob, p, act, dev, internal=False):
        self.jfa, self.prob, self.p, self.act = jfa, prob, p, act
        self.mx = p.dtype == "mxfp8" and not internal
        self.ws_f = jfa.workspace(prob, False, dev)
        self.bprob = prob
        if self.mx:
            self.bprob = jfa.jfa_problem.from_buffer_copy(prob)
            self.bprob.dtype = jfa.JFA_BF16
            H, dd = prob.heads, prob.head_dim
            u8 = dict(dtype=torch.uint8, device=dev)
            self.q8 = torch.empty(prob.total_q, H, dd, **u8)
            self.k8 = torch.empty(prob.total_kv, H, dd, **u8)
            self.v8 = torch.empty(prob.total_kv, H, dd, **u8)
            self.qs = torch.empty(prob.total_q, H, dd // 32, **u8)
            self.ks = torch.empty(prob.total_kv, H, dd // 32, **u8)
            self.vs = torch.empty(prob.total_kv // 32 + prob.batch, H, dd, **u8)
            bf = dict(dtype=torch.bfloat16, device=dev)
            self.qd = torch.empty(prob.total_q, H, dd, **bf)
            self.kd = torch.empty(prob.total_kv, H, dd, **bf)
            self.vd = torch.empty(prob.total_kv, H, dd, **bf)
        self.ws_b = jfa.workspace(self.bprob, True, dev)
        self.workspaces = (self.ws_f, self.ws_b)

    def forward(self, inp, qo, ko, bias, out, lse, stream):
        j, pr, causal = self.jfa, self.prob, self.p.causal
        if not self.mx:
            j.jfa_forward(pr, inp["q"], inp["k"], inp["v"], qo, ko, bias, self.act, causal, out, lse,
                          self.ws_f, stream=stream)
            return
        H, dd = pr.heads, pr.head_dim
        j.jfa_quantize_mxfp8_dequant(inp["q"], pr.total_q, H, dd, None, 0, 0, False, self.q8, self.qs,
                                     self.qd, stream=stream)
        j.jfa_quantize_mxfp8_dequant(inp["k"], pr.total_kv, H, dd, None, 0, 0, False, self.k8, self.ks,
                                     self.kd, stream=stream)
        j.jfa_quantize_mxfp8_dequant(inp["v"], pr.total_kv, H, dd, ko, pr.batch, pr.max_kv_len, True,
                                     self.v8, self.vs, self.vd, stream=stream)
        j.jfa_forward_mxfp8(pr, self.q8, self.qs, self.k8, self.ks, self.v8, self.vs, qo, ko, bias,
                            causal, out, lse, self.ws_f, stream=stream)

    def backward(self, inp, qo, ko, bias, out, lse, dq, dk, dv, stream):
        q, k, v = (self.qd, self.kd, self.vd) if self.mx else (inp["q"], inp["k"], inp["v"])
        self.jfa.jfa_backward(self.bprob, q, k, v, out, lse, inp["dout"], qo, ko, bias, self.act,
                              self.p.causal, dq, dk, dv, self.ws_b, stream=stream)


def e2e_leg(args, p, prob, act, dev, stream, jfa, flops_rank, world):
    """Same metric with pinned host inputs copied in and every result copied
    out inside the timed region, pipelined the way a training input loop is:
    two sets of device buffers, the inputs of step i+1 copied in (one copy
    stream) and the results of step i-1 copied out (another) while step i
    computes; every step still moves all of its inputs and results."""
    host_in = {n: getattr(p, n).contiguous().pin_memory() for n in ("q", "k", "v", "dout")}
    host_in["q_off"] = p.q_off.contiguous().pin_memory()
    host_in["kv_off"] = p.kv_off.contiguous().pin_memory()
    if p.bias is not None:
        host_in["bias"] = p.bias.contiguous().pin_memory()
    sets = []
    for _ in range(2):
        dev_in = {n: torch.empty_like(t, device=dev) for n, t in host_in.items()}
        out = torch.empty_like(dev_in["q"])
        lse = torch.empty(p.total_q, p.H, dtype=torch.float32, device=dev) if act == "softmax" else None
        dq, dk, dv = torch.empty_like(dev_in["q"]), torch.empty_like(dev_in["k"]), torch.empty_like(dev_in["v"])
        sets.append((dev_in, out, lse, dq, dk, dv))
    apass = AttentionPass(jfa, prob, p, act, dev, internal=args.mx_internal)
    # BlockAttention: block offsets rebuilt from each step's sequence offsets
    boffs = [torch.empty(prob.batch + 1, dtype=torch.int32, device=dev) for _ in range(2)]

    def results_of(st):
        _, out, lse, dq, dk, dv = st
        return [out, dq, dk, dv] + ([lse] if lse is not None else [])

    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in results_of(sets[0])]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in results_of(sets[0]))
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(nsteps):
        for i in range(nsteps):
            b = i % 2
            dev_in, out, lse, dq, dk, dv = sets[b]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(comp_done[b])       # step i-2 has finished reading set b
                for n, t in host_in.items():
                    dev_in[n].copy_(t, non_blocking=True)
                in_ready[b].record(up)
            stream.wait_event(in_ready[b])
            if i >= 2:
                stream.wait_event(out_free[b])        # results of step i-2 are out
            qo, ko = dev_in["q_off"], dev_in["kv_off"]
            if args.block:
                jfa.jfa_block_offsets(qo, p.B, p.total_q, args.block, boffs[b], stream=stream)
                qo = ko = boffs[b]
            apass.forward(dev_in, qo, ko, dev_in.get("bias"), out, lse, stream)
            apass.backward(dev_in, qo, ko, dev_in.get("bias"), out, lse, dq, dk, dv, stream)
            comp_done[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[b])
                for h, t in zip(host_out, results_of(sets[b])):
                    h.copy_(t, non_blocking=True)
                out_free[b].record(down)

    run(2)
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    s.record(stream)
    up.wait_event(s)
    run(args.e2e_steps)
    stream.wait_stream(down)
    stream.wait_stream(up)
    e.record(stream)
    torch.cuda.synchronize(dev)
    ms = s.elapsed_time(e) / args.e2e_steps
    ms, flops_all = aggregate_over_ranks(ms, flops_rank, dev, world)
    return {"value": flops_all / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": args.e2e_steps,
            "pipeline": "two buffer sets; inputs of step i+1 in and results of step i-1 out "
                        "on two copy streams while step i computes"}


if __name__ == "__main__":
    main()
