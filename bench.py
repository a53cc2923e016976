"""Benchmark: the NVFP4 DiT-block linear set at 2048^2 through libnvfp4.

One step = one pass of the whole hot path over one batch of 16896 tokens (16384 image + 512 text),
hidden 4608:
    quantise x_qkv (dynamic amax)  -> QKV GEMM [13824 x 4608] + bias + per-head q/k RMSNorm
    quantise x_attn                -> out-proj GEMM [4608 x 4608] + bias
    quantise x_ffn                 -> up GEMM [24576 x 4608] + gated SiLU + NVFP4 re-quantisation
    (up's NVFP4 output)            -> down GEMM [4608 x 12288] + residual + per-channel gate
Weights are quantised once before timing (they are static).  Every activation is 156 MB, larger
than the 126 MB L2, so each step streams its inputs from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One JSON line on rank 0.  Under torchrun each rank runs an independent replica on its own GPU (the
path has no exchange step); the time is the max over ranks and the value counts all ranks' work.
"""
from __future__ import annotations

import argparse
import datetime
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

from epilogue_gemm_nvfp4_b200 import workloads as W  # noqa: E402

METRIC = "fused NVFP4 linear TFLOPS and % of B200 dense FP4 peak; us per DiT-block linear set"
UNIT = "TFLOP/s"
WORKLOAD = "dit_block_linear_set_2048sq"
NOMINAL_FP4_TFLOPS = 9000.0   # NVIDIA's dense FP4 figure for B200
BF16_TO_FP4 = 4.0             # nominal dense FP4 / dense bf16 tensor-core rate (9 / 2.25)


#: the DRAM traffic of one full-size launch of the dominant kernel, written with its ncu capture
TRAFFIC_DATA = os.path.join(ROOT, "profiles", "nvfp4_gemm_up_dram_2048sq.json")


#: the sources the up-projection GEMM is built from: its device code and the host code that launches it
GEMM_SOURCES = ("ptx.cuh", "quantize.cuh", "gemm.cuh", "gemm_pair.cuh", "nvfp4_api.cu")

#: FP4 tensor-core rate of one SM: a 128 x 256 x 64 block-scaled MMA every 128 cycles
FP4_FLOP_PER_CLK_SM = 32768


def _code_only(text: str) -> str:
    """Source text without // comments, trailing blanks and empty lines: a comment edit leaves it unchanged."""
    lines = []
    for line in text.splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code:
            lines.append(code)
    return "\n".join(lines)


def library_sources_sha256():
    """sha256 over the code of the up GEMM's sources (GEMM_SOURCES, comments dropped): each file's name,
    then its code, in that order."""
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        h.update(name.encode())
        with open(os.path.join(ROOT, "epilogue_gemm_nvfp4_b200", "csrc", name)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()


def measured_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed capture record, or None when the
    library's sources have changed since those counters were taken."""
    try:
        with open(TRAFFIC_DATA) as fh:
            rec = json.load(fh)
        if rec.get("sources_sha256") != library_sources_sha256():
            return None
        return int(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"], hbm=d["hbm_gbs"], src="measured")
    return dict(bf16=1590.0, bf16_sus=1400.0, hbm=6650.0, src="fallback")


def layer_flops(M):
    H, F = W.HIDDEN, W.FFN
    return dict(qkv=2.0 * M * 3 * H * H, out=2.0 * M * H * H, up=2.0 * M * 2 * F * H, down=2.0 * M * H * F)


# ------------------------------------------------------------------------------------------
# distributed plumbing (replicas)
# ------------------------------------------------------------------------------------------

def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun env).  `gloo` runs the same plumbing on CPU (tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 10 ms while the timed region runs.

    The sampler is running (its first sample written) before the region starts.  Samples are matched to
    the region by their timestamps; a region shorter than the sampling interval may hold none, and then
    the samples just before and after it (same work, the warm-up and the steps after) stand in for it,
    which the summary says."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 10   # nvidia-smi keeps this rate on B200; a 44 ms timed region holds about four samples

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        deadline = time.time() + 5.0
        while self.proc is not None and time.time() < deadline and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)
        return self

    def start(self):
        self.t0 = datetime.datetime.now()

    def stop(self):
        self.t1 = datetime.datetime.now()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2 * self.INTERVAL_MS / 1000.0)  # one more sample after the region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        with open(self.path) as fh:
            lines = fh.readlines()
        os.unlink(self.path)
        return summarize_clock_samples(lines, self.t0, self.t1)


def summarize_clock_samples(lines, t0, t1):
    """Median SM clock, max clock, max power and the throttle reasons seen in the samples taken between
    t0 and t1 (datetimes), or in the nearest sample on each side when none falls in between."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            rows.append(dict(t=datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f"), sm=float(parts[2]),
                             smax=float(parts[3]), power=float(parts[4]), hw=parts[6], hwt=parts[7], swt=parts[8],
                             pcap=parts[9]))
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    window = "timed region"
    if t0 is not None and t1 is not None:
        inside = [r for r in rows if t0 <= r["t"] <= t1]
        if not inside:
            before = [r for r in rows if r["t"] < t0][-1:]
            after = [r for r in rows if r["t"] > t1][:1]
            inside = before + after
            window = "adjacent to the timed region (shorter than the sampling interval)"
        rows = inside or rows
    reasons = set()
    for r in rows:
        for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                        ("pcap", "sw_power_cap")):
            if r[k].lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
            "power_w_max": max(r["power"] for r in rows), "samples": len(rows), "window": window,
            "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# native arm
# ------------------------------------------------------------------------------------------

class BlockSet:
    """Device state of the DiT-block linear set: static NVFP4 weights, activations, outputs."""

    def __init__(self, seed=7, M=W.IMG_TOKENS_2K + W.PROMPT_T):
        from epilogue_gemm_nvfp4_b200 import binding as B
        self.B = B
        cases = W.block_2k(seed=seed, M=M)
        self.M = M
        self.cases = cases
        dev = torch.device("cuda")
        q, o, u, d = cases["qkv"], cases["out"], cases["up"], cases["down"]
        self.x = {k: cases[k].x.to(dev) for k in ("qkv", "out", "up")}
        self.wq = {k: B.quantize(cases[k].w.to(dev)) for k in ("qkv", "out", "up", "down")}
        self.bias = {k: cases[k].bias.to(dev) for k in ("qkv", "out")}
        ex = q.extras
        self.qk = dict(gamma_q=ex["gamma_q"].to(dev), gamma_k=ex["gamma_k"].to(dev), eps=ex["eps"],
                       q_col0=ex["q_col0"], k_col0=ex["k_col0"], qk_cols=ex["qk_cols"], head_dim=ex["head_dim"])
        self.res = d.extras["residual"].to(dev)
        self.gate = d.extras["gate"].to(dev)
        # activation NVFP4 buffers and outputs, allocated once
        self.aq = {k: B.QTensor.empty(M, W.HIDDEN) for k in ("qkv", "out", "up")}
        self.up_q = B.QTensor.empty(M, W.FFN)
        self.out = {"qkv": torch.empty(M, 3 * W.HIDDEN, dtype=torch.bfloat16, device=dev),
                    "out": torch.empty(M, W.HIDDEN, dtype=torch.bfloat16, device=dev),
                    "down": torch.empty(M, W.HIDDEN, dtype=torch.bfloat16, device=dev)}
        # static decode scale of the up projection's NVFP4 output, calibrated once on this input
        self.up_q.g.fill_(1.0)
        aq = B.quantize(self.x["up"], out=self.aq["up"])
        probe = B.linear(aq, self.wq["up"], "gated_silu")
        torch.cuda.synchronize()
        self.up_q.g.fill_(float(probe.abs().max().float().item()) / 2688.0)
        del probe
        torch.cuda.synchronize()

    def io_slot(self):
        """Second set of input / output buffers that shares this set's weights and NVFP4 scratch, so
        that the copies of one step can overlap the compute of another (the compute itself stays on
        one stream, so the quantised activations need no second copy)."""
        import copy
        s = copy.copy(self)
        s.x = {k: torch.empty_like(v) for k, v in self.x.items()}
        s.res = torch.empty_like(self.res)
        s.out = {k: torch.empty_like(v) for k, v in self.out.items()}
        return s

    def step(self, ev=None):
        """One pass of the hot path; `ev` (dict of event lists) brackets each op when given."""
        B = self.B

        def mark(name, i):
            if ev is not None:
                ev[name][i].record()
        mark("quant_qkv", 0); B.quantize(self.x["qkv"], out=self.aq["qkv"]); mark("quant_qkv", 1)
        mark("qkv", 0)
        B.linear(self.aq["qkv"], self.wq["qkv"], "qknorm", bias=self.bias["qkv"], out=self.out["qkv"], **self.qk)
        mark("qkv", 1)
        mark("quant_out", 0); B.quantize(self.x["out"], out=self.aq["out"]); mark("quant_out", 1)
        mark("out", 0); B.linear(self.aq["out"], self.wq["out"], "bias", bias=self.bias["out"], out=self.out["out"])
        mark("out", 1)
        mark("quant_up", 0); B.quantize(self.x["up"], out=self.aq["up"]); mark("quant_up", 1)
        mark("up", 0); B.linear(self.aq["up"], self.wq["up"], "gated_silu", out_fp4=self.up_q, want_bf16=False)
        mark("up", 1)
        mark("down", 0)
        B.linear(self.up_q, self.wq["down"], "resid_gate", residual=self.res, gate=self.gate, out=self.out["down"])
        mark("down", 1)

    LAUNCHES_PER_STEP = 3 * 2 + 4   # per activation: amax (which also writes g), quantise; four GEMMs


OPS = ("quant_qkv", "qkv", "quant_out", "out", "quant_up", "up", "down")


def run_native(args, ws, rank, local):
    from epilogue_gemm_nvfp4_b200 import binding as B
    B.load()
    bs = BlockSet()
    M = bs.M
    fl = layer_flops(M)
    step_flops = sum(fl.values())

    for _ in range(args.warmup):
        bs.step()
    torch.cuda.synchronize()
    B.check_device_error()

    # device-timed region: K steps, per-op events on the launching (current) stream
    ev = {k: [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
              for _ in range(args.steps)] for k in OPS}
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        clk.start()
        start.record()
        for i in range(args.steps):
            bs.step({k: ev[k][i] for k in OPS})
        stop.record()
        torch.cuda.synchronize()
        clk.stop()
    barrier(ws)
    B.check_device_error()
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local, ws)
    per_op = {k: statistics.mean(e[0].elapsed_time(e[1]) for e in ev[k]) for k in OPS}
    ms_step = ms / args.steps
    value = step_flops * ws / (ms_step * 1e-3) / 1e12

    # end to end through the public API with host buffers: every step copies its three activations and
    # the residual from pinned host memory to the device and its three bf16 outputs back.  The steps are
    # pipelined as a serving loop runs them: the copy-in of step i+1, the compute of step i and the
    # copy-out of step i-1 overlap on three streams, with two sets of device buffers.  The timed region
    # runs from the first copy-in to the last copy-out.
    host_in = {k: bs.x[k].cpu().pin_memory() for k in ("qkv", "out", "up")}
    host_res = bs.res.cpu().pin_memory()
    host_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in bs.out.items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + host_res.numel() * host_res.element_size()
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    e2e_steps = max(4, min(args.steps, 20))
    slots = [bs, bs.io_slot()]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n, timed):
        ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]  # copied in, computed, copied out
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            sl = slots[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev[i - 2][1])       # this slot's inputs are no longer read
                for k in host_in:
                    sl.x[k].copy_(host_in[k], non_blocking=True)
                sl.res.copy_(host_res, non_blocking=True)
                ev[i][0].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(ev[i][0])
                if i >= 2:
                    s_c.wait_event(ev[i - 2][2])        # this slot's outputs have been copied out
                sl.step()
                ev[i][1].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[i][1])
                for k in host_out:
                    host_out[k].copy_(sl.out[k], non_blocking=True)
                ev[i][2].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) if timed else 0.0
    e2e_run(2, False)
    barrier(ws)
    e2e_ms = max_over_ranks(e2e_run(e2e_steps, True), ws) / e2e_steps
    barrier(ws)

    pk = peaks()
    dominant = max(("qkv", "out", "up", "down"), key=lambda k: fl[k])
    achieved = fl[dominant] / (per_op[dominant] * 1e-3) / 1e12
    clocks = clk.summary()
    # the burst bf16 figure for a region under a second (the clock stays near its maximum there), the
    # sustained one for a region long enough to settle under the power cap
    sustained = ms > 1000.0
    peak_fp4 = (pk["bf16_sus"] if sustained else pk["bf16"]) * BF16_TO_FP4
    sm_count = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    at_clock = (FP4_FLOP_PER_CLK_SM * sm_count * clocks["sm_mhz"] * 1e6 / 1e12) if clocks.get("sm_mhz") else None
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 e2m1 x e4m3/16 -> fp32 acc", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M, "hidden": W.HIDDEN, "ffn": W.FFN, "heads": W.N_HEADS,
                   "head_dim": W.HEAD_DIM, "seed": 7, "parallelism": f"replicas x{ws}",
                   "l2": "inputs larger than L2 (each activation 156 MB)"},
        "us_per_block_linear_set": round(ms_step * 1e3, 1),
        "frac_of_nominal_fp4": round(value / ws / NOMINAL_FP4_TFLOPS, 4),
        "per_op_us": {k: round(v * 1e3, 1) for k, v in per_op.items()},
        "per_gemm_tflops": {k: round(fl[k] / (per_op[k] * 1e-3) / 1e12, 1) for k in ("qkv", "out", "up", "down")},
        "roofline": {"bound": "tensor",
                     "kernel": f"nvfp4_gemm_pair_kernel ({dominant}: gated SiLU + NVFP4 requant, CTA pairs)",
                     "achieved": round(achieved, 1), "peak": round(peak_fp4, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / peak_fp4, 4),
                     "peak_note": (f"{pk['src']} {'sustained' if sustained else 'burst'} bf16 "
                                   f"{pk['bf16_sus'] if sustained else pk['bf16']} x {BF16_TO_FP4} (nominal FP4/bf16 "
                                   f"ratio); the timed region ran {ms:.0f} ms"),
                     "frac_of_nominal_9pf": round(achieved / NOMINAL_FP4_TFLOPS, 4),
                     "peak_at_sampled_clock": round(at_clock, 1) if at_clock else None,
                     "frac_at_sampled_clock": round(achieved / at_clock, 4) if at_clock else None,
                     "at_clock_note": f"{FP4_FLOP_PER_CLK_SM} FLOP/clock/SM x {sm_count} SMs x the median sampled SM clock",
                     "traffic": measured_traffic(),
                     "traffic_note": "bytes per launch, ncu dram read+write of one full-size launch "
                                     "(profiles/nvfp4_gemm_up_dram_2048sq.json); null once the kernel sources change"},
        "quantize_roofline": None,
        "e2e": {"value": round(step_flops * ws / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipelined": "copy-in, compute and copy-out on three streams"},
        "gpu_launches": BlockSet.LAUNCHES_PER_STEP * args.steps,
    }
    qbytes = 2.5625 * M * W.HIDDEN
    qus = per_op["quant_qkv"] * 1e3
    q2bytes = 4.5625 * M * W.HIDDEN   # both passes: the amax read, then the quantise read and writes
    out["quantize_roofline"] = {"bound": "hbm", "kernel": "amax_scale_kernel + quantize_kernel (x [16896, 4608])",
                                "achieved": round(qbytes / (qus * 1e-6) / 1e9, 1), "peak": pk["hbm"], "unit": "GB/s",
                                "frac": round(qbytes / (qus * 1e-6) / 1e9 / pk["hbm"], 4),
                                "achieved_two_pass": round(q2bytes / (qus * 1e-6) / 1e9, 1),
                                "frac_two_pass": round(q2bytes / (qus * 1e-6) / 1e9 / pk["hbm"], 4),
                                "note": "achieved: the single-pass 2.5625 B/elem (2 B read, 0.5625 B written) over "
                                        "the whole dynamic-scale op; achieved_two_pass also counts the amax pass's "
                                        "2 B/elem read, which the dynamic scale needs because every element's code "
                                        "depends on the tensor amax and the 156 MB tensor exceeds L2"}
    out["clocks"] = clocks
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return out


# ------------------------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and the reference arm)
# ------------------------------------------------------------------------------------------

class OracleSample:
    """A bounded sample of the block workload for the oracle: `rows` tokens; every layer keeps whole
    heads / gate pairs and the full reduction width.  Weights are quantised once (static, untimed)."""

    def __init__(self, rows=64, seed=7):
        from oracle import nvfp4_oracle as O
        self.O = O
        rng = np.random.default_rng(seed)
        H, F, K = W.HIDDEN, W.FFN, W.HIDDEN
        f = lambda a: W.to_bf16(a).float().numpy()
        self.rows, self.rng, self.f = rows, rng, f
        w = {"qkv": f(W.normal(rng, (1536, K), 0.015)), "out": f(W.normal(rng, (512, K), 0.015)),
             "up": f(W.normal(rng, (1024, K), 0.015)), "down": f(W.normal(rng, (512, F), 0.01))}
        self.wq = {k: O.quantize(v) for k, v in w.items()}
        self.bias = {"qkv": f(W.normal(rng, (1536,), 0.01)), "out": f(W.normal(rng, (512,), 0.01))}
        self.gam = f(W.uniform(rng, (256,), 0.5, 1.5))
        self.gate = W.uniform(rng, (512,), 0.0, 1.0)
        self.flops = 2.0 * rows * K * (1536 + 512 + 1024) + 2.0 * rows * F * 512
        self.note = (f"{rows} tokens x (QKV 1536 + out 512 + up 1024 + down 512 weight rows), full K; "
                     "activation quantisation, GEMMs, epilogues and requant timed; weight quantisation not")

    def step(self):
        """Draw one batch of activations, then time the oracle's pass over it.  Returns seconds."""
        O, f, rng, rows = self.O, self.f, self.rng, self.rows
        x = {k: f(W.normal(rng, (rows, W.HIDDEN))) for k in ("qkv", "out", "up")}
        x_dn = f(W.normal(rng, (rows, W.FFN)))
        res = f(W.normal(rng, (rows, 512)))
        t0 = time.perf_counter()
        O.linear(O.quantize(x["qkv"]), self.wq["qkv"], "qknorm", bias=self.bias["qkv"], gamma_q=self.gam,
                 gamma_k=self.gam, eps=1e-6, q_col0=0, k_col0=512, qk_cols=512)
        O.linear(O.quantize(x["out"]), self.wq["out"], "bias", bias=self.bias["out"])
        O.linear(O.quantize(x["up"]), self.wq["up"], "gated_silu", out_g=np.float32(0.01))
        O.linear(O.quantize(x_dn), self.wq["down"], "resid_gate", residual=res, gate=self.gate)
        return time.perf_counter() - t0


def cpu_baseline(seconds=15.0):
    smp = OracleSample()
    dt = 0.0
    reps = 0
    while reps < 2 or dt < seconds:
        dt += smp.step()
        reps += 1
    return {"value": round(smp.flops * reps / dt / 1e12, 6), "unit": UNIT, "cores": torch.get_num_threads(),
            "kind": "oracle", "sample": f"{reps} x [{smp.note}]", "seconds": round(dt, 2)}


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    smp = OracleSample()
    note = smp.note
    times = [smp.step() for _ in range(args.warmup + args.steps)][args.warmup:]
    ms = statistics.mean(times) * 1e3
    val = smp.flops / (ms * 1e-3) / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle; fp32 quantiser steps)",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": W.IMG_TOKENS_2K + W.PROMPT_T, "hidden": W.HIDDEN,
                       "sample": note},
            "cpu_baseline": {"value": round(val, 6), "unit": UNIT, "cores": torch.get_num_threads(),
                             "kind": "oracle", "sample": note},
            "e2e": {"value": round(val, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------------------
# single-op mode: one layer of one workload, for per-config numbers and profiler captures
# ------------------------------------------------------------------------------------------

def op_case(name):
    """(description, setup) for one op; setup() returns a zero-argument callable running the op once
    (through the C ABI) and the op's algorithmic FLOPs or bytes."""
    from epilogue_gemm_nvfp4_b200 import binding as B
    dev = torch.device("cuda")

    def gemm(case, requant=False, with_amax=False):
        a = B.quantize(case.x.to(dev))
        w = B.quantize(case.w.to(dev))
        bias = case.bias.to(dev) if case.bias is not None else None
        ex = {}
        if case.epilogue == "qknorm":
            e = case.extras
            ex = dict(gamma_q=e["gamma_q"].to(dev), gamma_k=e["gamma_k"].to(dev), eps=e["eps"], q_col0=e["q_col0"],
                      k_col0=e["k_col0"], qk_cols=e["qk_cols"], head_dim=e["head_dim"])
        elif case.epilogue == "resid_gate":
            ex = dict(residual=case.extras["residual"].to(dev), gate=case.extras["gate"].to(dev))
        q = None
        if requant:
            q = B.QTensor.empty(case.M, case.n_out)
            q.g.fill_(0.01)
        out = torch.empty(case.M, case.n_out, dtype=torch.bfloat16, device=dev)
        if with_amax:  # the epilogue also publishes max |output| (the next call's delayed requant scale)
            ex["out_amax"] = torch.zeros(1, dtype=torch.float32, device=dev)
        fn = lambda: B.linear(a, w, case.epilogue, bias=bias, out=out if q is None else None, out_fp4=q,
                              want_bf16=q is None, **ex)
        return fn, W.flops(case), "TFLOP/s"

    def quant(rows, cols, static=False):
        x = W.to_bf16(W.normal(np.random.default_rng(0), (rows, cols))).to(dev)
        q = B.QTensor.empty(rows, cols)
        q.g.fill_(3.0 / 2688.0)
        return (lambda: B.quantize(x, out=q, static=static)), 2.5625 * rows * cols, "GB/s (2.5625 B/elem)"

    def fakeq(rows, cols, static=False):
        x = W.to_bf16(W.normal(np.random.default_rng(0), (rows, cols))).to(dev)
        y = torch.empty(rows, cols, dtype=torch.bfloat16, device=dev)
        scale = torch.full((1,), 3.0 / 2688.0, dtype=torch.float32, device=dev)
        return (lambda: B.fake_quantize(x, y=y, scale=scale, static=static)), 4.0 * rows * cols, "GB/s (4 B/elem)"

    def gemm_i8(case, requant=False):
        a = B.int8_quantize(case.x.to(dev))
        w = B.int8_quantize(case.w.to(dev))
        bias = case.bias.to(dev) if case.bias is not None else None
        ex = {}
        if case.epilogue == "qknorm":
            e = case.extras
            ex = dict(gamma_q=e["gamma_q"].to(dev), gamma_k=e["gamma_k"].to(dev), eps=e["eps"], q_col0=e["q_col0"],
                      k_col0=e["k_col0"], qk_cols=e["qk_cols"], head_dim=e["head_dim"])
        elif case.epilogue == "resid_gate":
            ex = dict(residual=case.extras["residual"].to(dev), gate=case.extras["gate"].to(dev))
        q = None
        if requant:
            q = B.QTensor.empty(case.M, case.n_out)
            q.g.fill_(0.01)
        out = torch.empty(case.M, case.n_out, dtype=torch.bfloat16, device=dev)
        fn = lambda: B.int8_linear(a, w, case.epilogue, bias=bias, out=out if q is None else None, out_fp4=q,
                                   want_bf16=q is None, **ex)
        return fn, W.flops(case), "TOP/s (int8)"

    def int8_quant(rows, cols):
        x = W.to_bf16(W.normal(np.random.default_rng(0), (rows, cols))).to(dev)
        mult = torch.rand(cols, dtype=torch.float32, device=dev) + 0.5
        out = B.Int8Tensor.empty(rows, cols)
        return (lambda: B.int8_quantize(x, mult, out=out)), 3.0 * rows * cols + 4.0 * (rows + cols), "GB/s (3 B/elem)"

    def adaln(static=False):
        case = W.adaln_2k()
        x, sh, sc = case.x.to(dev), case.shift[0].to(dev), case.scale[0].to(dev)
        rows, cols = case.x.shape
        q = B.QTensor.empty(rows, cols)
        q.g.fill_(3.0 / 2688.0)
        fn = lambda: B.adaln_quantize(x, sh, sc, eps=case.eps, out=q, static=static)
        return fn, 2.5625 * rows * cols + 4.0 * cols, "GB/s (2.5625 B/elem)"

    def amax(rows, cols):
        x = W.to_bf16(W.normal(np.random.default_rng(0), (rows, cols))).to(dev)
        o = torch.empty(1, dtype=torch.float32, device=dev)
        return (lambda: B.amax(x, out=o)), 2.0 * rows * cols, "GB/s (2 B/elem)"

    M1 = W.IMG_TOKENS_1K + W.PROMPT_T
    M2 = W.IMG_TOKENS_2K + W.PROMPT_T
    table = {
        "tiny": lambda: gemm(W.tiny()),
        "qkv_1k": lambda: gemm(W.qkv_1k()),
        "up_1k": lambda: gemm(W.case_ffn_up(M1), requant=True),
        "up_1k_amax": lambda: gemm(W.case_ffn_up(M1), requant=True, with_amax=True),
        "down_1k": lambda: gemm(W.case_ffn_down(M1)),
        "text_512": lambda: gemm(W.text_proj(W.PROMPT_T)),
        "text_1941": lambda: gemm(W.text_proj(W.LONG_PROMPT_T)),
        "text_512z": lambda: gemm(W.text_proj(W.PROMPT_T, zero_rows=W.IMG_TOKENS_1K)),
        "out_2k": lambda: gemm(W.case_bias(M2, W.HIDDEN, W.HIDDEN, seed=8, w_std=0.015)),
        "quant_1k": lambda: quant(M1, W.HIDDEN),
        "quant_2k": lambda: quant(M2, W.HIDDEN),
        "quant_text": lambda: quant(W.HIDDEN, W.TEXT_K),
        "quant_2k_static": lambda: quant(M2, W.HIDDEN, static=True),
        "fakeq_2k": lambda: fakeq(M2, W.HIDDEN),
        "fakeq_2k_static": lambda: fakeq(M2, W.HIDDEN, static=True),
        "quant_text_static": lambda: quant(W.HIDDEN, W.TEXT_K, static=True),
        "amax_2k": lambda: amax(M2, W.HIDDEN),
        "w8a8_qkv_1k": lambda: gemm_i8(W.qkv_1k()),
        "w8a8_up_1k": lambda: gemm_i8(W.case_ffn_up(M1), requant=True),
        "w8a8_down_1k": lambda: gemm_i8(W.case_ffn_down(M1)),
        "w8a8_out_2k": lambda: gemm_i8(W.case_bias(M2, W.HIDDEN, W.HIDDEN, seed=8, w_std=0.015)),
        "int8_quant_2k": lambda: int8_quant(M2, W.HIDDEN),
        "adaln_2k": lambda: adaln(),
        "adaln_2k_static": lambda: adaln(static=True),
    }
    return table[name]


def run_op(args):
    from epilogue_gemm_nvfp4_b200 import binding as B
    torch.cuda.set_device(0)
    fn, work, unit = op_case(args.op)()
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    B.check_device_error()
    # back-to-back launches between two events: the host enqueues ahead of the device, so the mean
    # is the device time per call (per-call events would also count host launch gaps)
    reps = []
    for _ in range(3):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            fn()
        e.record()
        torch.cuda.synchronize()
        reps.append(s.elapsed_time(e) / args.steps)
    B.check_device_error()
    med = sorted(reps)[1]
    scale = 1e12 if unit.startswith(("TFLOP", "TOP")) else 1e9
    return {"op": args.op, "mean_us": round(med * 1e3, 2), "min_us": round(min(reps) * 1e3, 2),
            "value": round(work / (med * 1e-3) / scale, 1), "unit": unit, "steps": args.steps}


#: plain products of the benchmarked shapes (M, N, K) for the library comparison
LIBRARY_SHAPES = {
    "out_2k": (16896, 4608, 4608),
    "qkv_2k": (16896, 13824, 4608),
    "up_2k": (16896, 24576, 4608),
    "down_2k": (16896, 4608, 12288),
    "qkv_1k": (4608, 13824, 4608),
    "down_1k": (4608, 4608, 12288),
    "text_512": (512, 4608, 53248),
}


def run_library_comparison(args):
    """Our fused linear (zero bias, bf16 out) beside cuBLASLt's NVFP4 GEMM (torch scaled_mm, block-16
    E4M3 scales plus the fp32 tensor scales) on the same quantised operands: the scale layout of this
    library is the 32 x 4 x 4 atom layout cuBLASLt reads, so both consume the same bytes.  Prints one
    JSON line per shape: device times (median of 3 x args.steps back-to-back launches) and the largest
    difference between the two bf16 outputs."""
    import torch.nn.functional as F
    from epilogue_gemm_nvfp4_b200 import binding as B
    torch.cuda.set_device(0)
    dev = "cuda"

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        reps = []
        for _ in range(3):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            for _ in range(args.steps):
                fn()
            e.record()
            torch.cuda.synchronize()
            reps.append(s.elapsed_time(e) / args.steps)
        return sorted(reps)[1] * 1e3

    for name, (M, N, K) in LIBRARY_SHAPES.items():
        gen = torch.Generator(device=dev).manual_seed(1)
        xq = B.quantize(torch.randn(M, K, device=dev, dtype=torch.bfloat16, generator=gen))
        wq = B.quantize(torch.randn(N, K, device=dev, dtype=torch.bfloat16, generator=gen) * 0.02)
        bias = torch.zeros(N, device=dev, dtype=torch.bfloat16)
        out = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        flop = 2.0 * M * N * K
        res = {"compare": "cublaslt_nvfp4", "shape": name, "M": M, "N": N, "K": K}
        ours_us = timed(lambda: B.linear(xq, wq, "bias", bias=bias, out=out))
        B.check_device_error()
        res.update(ours_us=round(ours_us, 2), ours_tflops=round(flop / ours_us / 1e6, 1))
        try:
            sa = [xq.scales.view(torch.float8_e4m3fn), xq.g]
            sb = [wq.scales.view(torch.float8_e4m3fn), wq.g]
            recipe = [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise]
            swz = [F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE]
            a4 = xq.codes.view(torch.float4_e2m1fn_x2)
            b4 = wq.codes.view(torch.float4_e2m1fn_x2).t()
            lib = lambda: F.scaled_mm(a4, b4, sa, recipe, sb, recipe, swizzle_a=swz, swizzle_b=swz,
                                      output_dtype=torch.bfloat16)
            y = lib()
            res["max_abs_diff"] = float((y.float() - out.float()).abs().max())
            res["identical"] = bool(torch.equal(y, out))
            del y
            lib_us = timed(lib)
            res.update(cublaslt_us=round(lib_us, 2), cublaslt_tflops=round(flop / lib_us / 1e6, 1),
                       ours_over_cublaslt=round(lib_us / ours_us, 3))
        except Exception as e:  # a torch without the NVFP4 path: report, do not fail
            res["cublaslt"] = f"unavailable: {type(e).__name__}: {str(e)[:200]}"
        print(json.dumps(res), flush=True)
        del xq, wq, out
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default=None, help="time one op instead of the block step (profiling / per-config)")
    ap.add_argument("--compare-cublaslt", action="store_true",
                    help="time the plain NVFP4 products of the benchmarked shapes beside cuBLASLt's NVFP4 GEMM")
    args = ap.parse_args()
    if args.compare_cublaslt:
        run_library_comparison(args)
        return
    if args.op is not None:
        for name in args.op.split(","):
            args.op = name
            print(json.dumps(run_op(args)), flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    ws, rank, local = dist_init()
    res = run_native(args, ws, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
