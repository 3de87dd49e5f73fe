"""Benchmark of the BinaryAttention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {binattn,reference}]
                    [--workload dit_xl_1024] [--engine auto|tc|popc_tc|simt]

One step = the whole hot path over one batch: binattn_pack(Q), binattn_pack(K)
and binattn_forward, on DiT-XL/2 @1024px-shaped synthetic inputs (B=2, H=16,
N=4096, d=72) with the dense bf16 bias [16, 4096, 4096] resident on the device.
The same step without the bias is timed as well and reported under "no_bias".

Timing: W untimed warm-up steps (plus about a second of untimed steps, during
which clocks are sampled), then K steps, each between a pair of CUDA events on
the launching stream, with a 256 MiB write between steps so that L2 (126 MB)
starts cold for every step. Barrier + synchronize bracket the timed region; the
step time is the max over ranks. With N > 1 every rank runs its own batch
(weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (the reference implementation of this
path) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
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

from diffusion_transformers_b200.synthetic import WORKLOADS, make_inputs  # noqa: E402

METRIC = "BinaryAttention fwd ms & effective TFLOPS at DiT-XL N=4096; % of roofline"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="binattn", choices=["binattn", "reference"])
    ap.add_argument("--workload", default="dit_xl_1024", choices=sorted(WORKLOADS))
    ap.add_argument("--engine", default="auto")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="with N > 1: none = every rank runs its own batch (weak scaling); heads = one "
                         "batch split by heads, rank r holding only its heads' Q, K, V and bias (strong "
                         "scaling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the bounded oracle sample")
    ap.add_argument("--profile-once", action="store_true",
                    help="run --warmup plain steps (with bias) and exit: the command profiled by ncu")
    ap.add_argument("--no-bias", action="store_true", help="with --profile-once: steps without bias")
    ap.add_argument("--profile-path", default="dense", choices=["dense", "int8", "relpos", "sample"],
                    help="with --profile-once: the forward call the steps make (dense or no bias, the 8-bit P.V "
                         "forward, the position-sensitive bias, one dense bias per batch entry)")
    ap.add_argument("--batch", type=int, default=None,
                    help="with --profile-once: replace the workload's batch B (a small case for multi-pass "
                         "ncu captures)")
    return ap.parse_args()


def workload_config(w, with_bias=True):
    return {
        "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d}, bf16 Q/K/V, "
                    + (f"dense bf16 bias [{w.H},{w.N},{w.N}]" if with_bias else "no bias"),
        "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bias": with_bias,
        "step": "pack(Q) + pack(K) + forward",
        "l2": "flushed between timed steps (256 MiB write)",
    }


def algorithmic(w, with_bias=True, bias_per_sample=False):
    """Per-launch algorithmic work of the forward kernel (one (b,h,i,j) pair =
    2d binary ops for QK, 2d flops for P.V). bias_per_sample: one dense bias
    per batch entry ([B, H, N, N], the context-aware form) instead of [H, N, N]."""
    BH, N, d = w.B * w.H, w.N, w.d
    pairs = BH * N * N
    W = (d + 31) // 32
    bytes_ = (2 * BH * N * W * 4          # q_bits, k_bits
              + 2 * BH * N * 4            # alpha_q, alpha_k
              + 2 * BH * N * d * 2        # V read, O written
              + ((BH if bias_per_sample else w.H) * N * N * 2 if with_bias else 0))  # bias, once
    pack_bytes = 2 * (BH * N * d * 2 + BH * N * W * 4 + BH * N * 4)
    return dict(pairs=pairs, qk_ops=2 * d * pairs, pv_flops=2 * d * pairs,
                eff_flops=4 * d * pairs, bytes=bytes_, pack_bytes=pack_bytes)


def algorithmic_backward(w):
    """Algorithmic work of one backward call with the dense bias: the packed Q
    and K, alphas, V and dO read once, the bias read once, dV, ds, dt (fp32)
    and dbias (fp32, summed over b) written once; one binary QK^T recomputed
    (2d ops per pair) and four products of the P.V kind (dP, dV, ds, dt: 2d
    flops per pair each)."""
    BH, N, d = w.B * w.H, w.N, w.d
    pairs = BH * N * N
    W = (d + 31) // 32
    bytes_ = (2 * BH * N * W * 4 + 2 * BH * N * 4 + 2 * BH * N * d * 2 + w.H * N * N * 2
              + 3 * BH * N * d * 4 + w.H * N * N * 4)
    return dict(pairs=pairs, qk_ops=2 * d * pairs, pv_like_flops=8 * d * pairs, bytes=bytes_)


# The binary QK^T runs on tcgen05.mma kind::f8f6f4 with e4m3 +-1 operands. Its
# dense rate is twice the bf16 rate (NVIDIA's nominal 4.5 against 2.25 PFLOP/s
# per GPU; on this part an e4m3 M=128 N=128 K=32 MMA and a bf16 M=128 N=128
# K=16 MMA both take 64 cycles), so its peak is 2x the measured bf16 figure.
E4M3_OVER_BF16 = 2.0
MUFU_EXP_PER_CLK_PER_SM = 16  # ex2 throughput of the special-function unit


def roofline_terms(w, with_bias, peaks, n_sm=148, sm_mhz=None, bias_per_sample=False):
    """Roofline of one forward call: T_roof = max(T_mem, T_QK + T_PV), with
    T_mem = algorithmic bytes / HBM peak, T_PV = P.V flops / bf16 peak and
    T_QK = binary QK ops / e4m3 peak (the pipe the scores run on). The exp
    floor (one ex2 per pair on the special-function unit) is reported beside
    it; it is not part of T_roof."""
    a = algorithmic(w, with_bias, bias_per_sample)
    bf16 = peaks["bf16_tflops"] * 1e12
    e4m3 = E4M3_OVER_BF16 * bf16
    t_mem = a["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_pv = a["pv_flops"] / bf16
    t_qk = a["qk_ops"] / e4m3
    t_tensor = t_pv + t_qk
    clk = (sm_mhz or peaks.get("sm_max_mhz") or 1965.0) * 1e6
    t_mufu = a["pairs"] / (MUFU_EXP_PER_CLK_PER_SM * n_sm * clk)
    return dict(t_mem=t_mem, t_pv=t_pv, t_qk=t_qk, t_tensor=t_tensor, t_roof=max(t_mem, t_tensor),
                t_mufu=t_mufu, bound="hbm" if t_mem >= t_tensor else "tensor",
                tensor_peak_tflops=(a["qk_ops"] + a["pv_flops"]) / t_tensor / 1e12, work=a)


def roofline_line(w, with_bias, peaks, fwd_s, n_sm=148, sm_mhz=None, bias_per_sample=False):
    """The bench line's roofline object for a forward call of fwd_s seconds:
    frac = T_roof / fwd_s. Bound hbm: achieved = algorithmic bytes / time
    against the HBM peak. Bound tensor: achieved = (QK ops + P.V flops) / time
    against the blended peak (QK ops + P.V flops) / (T_QK + T_PV)."""
    r = roofline_terms(w, with_bias, peaks, n_sm, sm_mhz, bias_per_sample)
    a = r["work"]
    if r["bound"] == "hbm":
        achieved, peak, unit = a["bytes"] / fwd_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = (a["qk_ops"] + a["pv_flops"]) / fwd_s / 1e12, r["tensor_peak_tflops"], "TFLOP/s"
    return {"bound": r["bound"], "achieved": round(achieved, 2), "peak": round(peak, 2), "unit": unit,
            "frac": round(r["t_roof"] / fwd_s, 4),
            "t_roof_us": round(r["t_roof"] * 1e6, 2), "t_mem_us": round(r["t_mem"] * 1e6, 2),
            "t_qk_us": round(r["t_qk"] * 1e6, 2), "t_pv_us": round(r["t_pv"] * 1e6, 2),
            "t_exp_floor_us": round(r["t_mufu"] * 1e6, 2),
            "exp_floor_frac": round(r["t_mufu"] / fwd_s, 4)}


# DRAM traffic of one forward call from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum summed over the launches the call makes at dit_xl_1024
# with bias: the full-wave launch, the key-split tail launch and the combine; the
# summary is profiles/fwd_tc2_dit_xl_1024_bias.md; the same call with one bias per
# batch entry was captured on earlier sources, profiles/sample_bias_dit_xl_1024.md),
# valid only for the kernel
# sources it was taken on: any change to their code turns the reported traffic
# back into null. The digest covers the code only (comments removed, runs of
# white space collapsed), so an edit of a comment keeps the capture valid.
NCU_TRAFFIC = {
    "sources_sha256": "83b3d65fe546d7e5c9b94a48d41a5bf70cd6c61a101ce6082a566e9918cb02a2",
    "bytes_per_call": {"dit_xl_1024/bias": 588_474_624},
}

_C_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/', re.S)


def code_only(text):
    """C/C++/CUDA source with comments removed and white space collapsed."""
    kept = _C_TOKENS.sub(lambda m: " " if m.group(0)[0] == "/" else m.group(0), text)
    return " ".join(kept.split())


def kernel_sources_digest(root=ROOT):
    import hashlib
    csrc = os.path.join(root, "diffusion_transformers_b200", "csrc")
    h = hashlib.sha256()
    paths = [os.path.join(csrc, n) for n in sorted(os.listdir(csrc)) if n.endswith((".cu", ".cuh", ".h"))]
    paths.append(os.path.join(root, "include", "binattn.h"))
    for path in paths:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + b"\0" + code_only(f.read()).encode())
    return h.hexdigest()


def ncu_traffic(key):
    if kernel_sources_digest() != NCU_TRAFFIC["sources_sha256"]:
        return None
    return NCU_TRAFFIC["bytes_per_call"].get(key)


def percentile(xs, q):
    """Linearly interpolated q-quantile (0 <= q <= 1) of a non-empty sequence."""
    s = sorted(xs)
    pos = q * (len(s) - 1)
    lo = int(math.floor(pos))
    hi = min(lo + 1, len(s) - 1)
    return s[lo] + (s[hi] - s[lo]) * (pos - lo)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained"),
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), util=float(parts[4]),
                                 reasons=[n for n, v in zip(
                                     ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                      "sw_power_cap"), parts[5:9]) if v.lower() == "active"]))
            except ValueError:
                continue
        loaded = [r for r in rows if r["util"] > 0] or rows
        if not loaded:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({x for r in loaded for x in r["reasons"]})
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in loaded), "reasons": reasons,
                "samples": len(loaded)}


# ------------------------------------------------------------ oracle (CPU)
def cpu_oracle_sample(w, with_bias, target_s, inp=None):
    """Time the oracle on a bounded sample of query rows of the workload and
    extrapolate linearly to one whole step (pack is part of the oracle's prep)."""
    import oracle
    orc = oracle.get()
    if inp is None:
        inp = make_inputs(w, with_bias=with_bias)
    T = w.B * w.H * w.N
    rng = np.random.default_rng(123)
    bias = inp["bias"] if with_bias else None

    def run(n):
        rows = rng.integers(0, T, size=n)
        t0 = time.perf_counter()
        orc.forward_rows(inp["q"], inp["k"], bias, inp["v"], inp["softmax_scale"], rows)
        return time.perf_counter() - t0

    # t(n) = a + b n: a = signs and scales of every token (done once per call),
    # b = one query row's scores, softmax and P.V. Two sizes fix a and b.
    n1 = 256
    t1 = run(n1)
    n2 = n1 * 4
    t2 = run(n2)
    b = max((t2 - t1) / (n2 - n1), 1e-9)
    a = max(t1 - b * n1, 0.0)
    n3 = int(min(T, max(n2, (target_s - a) / b)))
    t3 = run(n3)
    b3 = max((t3 - a) / n3, 1e-9)
    ms = (a + b3 * T) * 1e3
    return dict(value=ms, unit="ms", cores=orc.num_threads(), kind="oracle",
                sample=f"{n3} of {T} query rows ({t3:.1f} s; per-call token prep {a:.2f} s, "
                       f"{b3 * 1e3:.3f} ms per row), extrapolated to all rows as prep + rows x per-row")


def cpu_oracle_all(skip, target_s=1.5, single_core=("tiny", "deit_b")):
    """The oracle on every other workload (with its bias), all host cores, a
    bounded sample of about target_s each; single-core as well on the small
    ones. Reported beside the GPU numbers, never timed against them."""
    import oracle
    orc = oracle.get()
    cores = orc.num_threads()
    out = {}
    for name in sorted(WORKLOADS):
        if name == skip:
            continue
        w = WORKLOADS[name]
        inp = make_inputs(w, with_bias=True)
        r = cpu_oracle_sample(w, True, target_s, inp)
        out[name] = {"ms": round(r["value"], 3), "cores": r["cores"], "sample": r["sample"]}
        if name in single_core:
            orc.set_num_threads(1)
            try:
                r1 = cpu_oracle_sample(w, True, target_s, inp)
            finally:
                orc.set_num_threads(cores)
            out[name]["single_core_ms"] = round(r1["value"], 3)
    return out


# ------------------------------------------------------------------ ranks
def rank_seed(w, rank):
    """Every rank draws its own batch of the workload (weak scaling): rank 0
    uses the workload's seed, rank r the seed + 1000 r."""
    return w.seed + 1000 * rank


def max_over_ranks_of(x, world, device):
    """Max of a per-rank scalar over all ranks (the step time of the job is
    that of its slowest rank). Every rank must call it, in the same order."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_units(units_per_rank, world):
    """Units processed by the whole job in one step: every rank processes its
    own full batch, no data-path collective."""
    return units_per_rank * world


def run_reference(args, w, rank):
    """The reference arm: the oracle on the host cores, W untimed then K timed
    steps. Each step times a bounded sample of query rows of the workload and
    extrapolates it to the whole workload (prep + rows x per-row, calibrated
    once); the samples are sized so that the whole run takes about 150 s."""
    if rank != 0:
        return
    import oracle
    orc = oracle.get()
    inp = make_inputs(w, with_bias=True)
    T = w.B * w.H * w.N
    rng = np.random.default_rng(123)

    def run(n):
        rows = rng.integers(0, T, size=n)
        t0 = time.perf_counter()
        orc.forward_rows(inp["q"], inp["k"], inp["bias"], inp["v"], inp["softmax_scale"], rows)
        return time.perf_counter() - t0

    n1, n2 = 256, 1024
    t1, t2 = run(n1), run(n2)
    b = max((t2 - t1) / (n2 - n1), 1e-9)
    a = max(t1 - b * n1, 0.0)
    per_step = max(0.5, min(args.cpu_seconds, 150.0 / max(args.steps + args.warmup, 1)))
    n = int(min(T, max(n2, (per_step - a) / b)))
    steps_ms = []
    for i in range(args.warmup + args.steps):
        t = run(n)
        if i >= args.warmup:
            steps_ms.append((a + max(t - a, 1e-9) / n * T) * 1e3)
    value = sum(steps_ms) / len(steps_ms)
    sample = (f"{n} of {T} query rows per step ({per_step:.1f} s target), extrapolated to all rows as "
              f"prep ({a:.2f} s) + rows x per-row; {args.warmup} untimed, {args.steps} timed steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": value,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, True),
        "cpu_baseline": {"value": value, "unit": "ms", "cores": orc.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU
def step_launches(w, with_bias, engine="auto"):
    """Kernels of one step: two packs, then the forward: one launch, or with the
    workspace path a bias-padding launch (N % 8 != 0) and, for a short last wave
    of 256-row pairs, the split launch and the combine kernel."""
    import torch
    n = 2 + 1
    if engine != "auto" or w.d % 8 or w.d > 80:
        return n
    if with_bias and w.N % 8:
        n += 1
    nsm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    pairs = w.B * w.H * (-(-w.N // 256))
    tail = pairs - pairs // nsm * nsm
    if pairs // nsm and tail and 2 * tail <= nsm and -(-w.N // 64) >= 32:
        n += 2
    return n


def time_configs(names, args, rank, world, dev, stream, peaks, flush, max_over_ranks):
    """Forward (with the dense bias) and whole-step times of other workloads:
    each one seeded and synthetic, timed over min(steps, 10) steps with a cold
    L2, max over ranks. Every rank runs the same list in the same order."""
    import torch
    from diffusion_transformers_b200 import binattn

    def to_dev(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(x).to(dev)

    rows = []
    steps = max(1, min(args.steps, 10))
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    for name in names:
        w = WORKLOADS[name]
        inp = make_inputs(w, with_bias=True, seed=rank_seed(w, rank))
        q, k, v, bias = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), to_dev(inp["bias"])
        scale = inp["softmax_scale"]
        qb, aq = binattn.pack(q, stream=stream)
        kb, ak = binattn.pack(k, stream=stream)
        out = torch.empty_like(v)
        # bias rows that are not TMA rows (N % 8 != 0): padded copy in a workspace
        need = binattn.workspace_bytes(w.B, w.H, w.N, w.d, True) if args.engine == "auto" else 0
        ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None

        def fwd():
            if ws is not None:
                binattn.forward_ws(qb, kb, aq, ak, bias, v, scale, workspace=ws, out=out, stream=stream)
            else:
                binattn.forward(qb, kb, aq, ak, bias, v, scale, out=out, engine=args.engine, stream=stream)

        for _ in range(3):
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            fwd()
        torch.cuda.synchronize()
        ev = []
        for _ in range(steps):
            flush.fill_(1)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            e[1].record(stream)
            fwd()
            e[2].record(stream)
            ev.append(e)
        torch.cuda.synchronize()
        binattn.device_status(stream)
        step_ms = max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in ev) / steps)
        fwd_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / steps)
        a = algorithmic(w, True)
        t_roof = roofline_terms(w, True, peaks, n_sm)["t_roof"]
        row = {"workload": name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bias": True,
               "call": "binattn_forward_ws" if ws is not None else "binattn_forward",
               "forward_ms": round(fwd_ms, 5), "step_ms": round(step_ms, 5),
               "effective_tflops": round(a["eff_flops"] / (fwd_ms * 1e-3) / 1e12, 2),
               "roofline_frac": round(t_roof / (fwd_ms * 1e-3), 4)}
        # The bias is a learned parameter: stored once with padded rows, the call
        # reads it as it is (binattn_forward_bias_ld_ws) instead of padding it.
        if args.engine == "auto" and w.N % 8 and w.d % 8 == 0 and w.d <= 80:
            stored = binattn.pad_bias(bias)
            wsl = torch.empty(max(16, binattn.lib().binattn_forward_bias_ld_workspace_bytes(
                w.B, w.H, w.N, w.d, stored.shape[2])), dtype=torch.uint8, device=dev)
            fl = lambda: binattn.forward_bias_ld_ws(qb, kb, aq, ak, stored, v, scale, workspace=wsl, out=out,
                                                    stream=stream)
            for _ in range(3):
                fl()
            torch.cuda.synchronize()
            evl = []
            for _ in range(steps):
                flush.fill_(1)
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(stream)
                fl()
                e[1].record(stream)
                evl.append(e)
            torch.cuda.synchronize()
            binattn.device_status(stream)
            fl_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evl) / steps)
            row["stored_padded_bias"] = {"call": "binattn_forward_bias_ld_ws", "forward_ms": round(fl_ms, 5),
                                         "roofline_frac": round(t_roof / (fl_ms * 1e-3), 4)}
            del stored, wsl
        rows.append(row)
        del q, k, v, bias, qb, kb, aq, ak, out, ws
    return rows


def rank_inputs(w, rank, world, shard_mode):
    """This rank's workload and inputs. Replicas: the whole workload on its own
    seed. Heads: one batch (the workload's seed on every rank) of which this
    rank holds heads head_range(H, world, rank) only, bias slice included."""

    from diffusion_transformers_b200 import shard
    if shard_mode == "heads" and world > 1:
        inp = shard.shard_inputs(make_inputs(w, with_bias=True, seed=w.seed), world, rank)
        return dataclasses.replace(w, H=inp["H"]), inp
    return w, make_inputs(w, with_bias=True, seed=rank_seed(w, rank))


def run_gpu(args, w_job, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from diffusion_transformers_b200 import binattn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()

    sharded = args.shard == "heads" and world > 1
    w, inp = rank_inputs(w_job, rank, world, args.shard)

    def to_dev(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(x).to(dev)

    q, k, v, bias = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), to_dev(inp["bias"])
    scale = inp["softmax_scale"]
    B, H, N, d = w.B, w.H, w.N, w.d
    W = (d + 31) // 32
    qb = torch.empty((B, H, N, W), dtype=torch.int32, device=dev)
    kb = torch.empty_like(qb)
    aq = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ak = torch.empty_like(aq)
    out = torch.empty_like(v)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    # binattn_forward_ws with a workspace allocated here, outside every timed
    # region (it splits a short last wave of row pairs by key halves);
    # binattn_forward when the shape needs no workspace or an engine is forced.
    ws = {}
    for key, has_bias in (("bias", True), ("no_bias", False)):
        need = binattn.workspace_bytes(B, H, N, d, has_bias) if args.engine == "auto" else 0
        ws[key] = torch.empty(need, dtype=torch.uint8, device=dev) if need else None

    def fwd(b):
        w = ws["bias" if b is not None else "no_bias"]
        if w is not None:
            binattn.forward_ws(qb, kb, aq, ak, b, v, scale, workspace=w, out=out, stream=stream)
        else:
            binattn.forward(qb, kb, aq, ak, b, v, scale, out=out, engine=args.engine, stream=stream)

    def step(b):
        binattn.pack(q, qb, aq, stream)
        binattn.pack(k, kb, ak, stream)
        fwd(b)

    def timed(b, steps, fwd_only_events=None):
        """Per-step events; returns (step_ms list, forward_ms list)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1, e2 in ev:
            flush.fill_(1)
            e0.record(stream)
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            e1.record(stream)
            fwd(b)
            e2.record(stream)
        torch.cuda.synchronize()
        return ([e0.elapsed_time(e2) for e0, _, e2 in ev], [e1.elapsed_time(e2) for _, e1, e2 in ev])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        return max_over_ranks_of(x, world, dev)

    if args.profile_once:
        b = None if args.no_bias else bias
        if args.profile_path == "int8":
            iws = torch.empty(max(16, binattn.int8_workspace_bytes(B, H, N, d, b is not None)), dtype=torch.uint8,
                              device=dev)
            call = lambda: binattn.forward_int8(qb, kb, aq, ak, b, v, scale, workspace=iws, out=out, stream=stream)
        elif args.profile_path == "relpos":
            g = int(round(math.sqrt(N)))
            if g * g != N:
                raise SystemExit("--profile-path relpos needs a square patch grid (N = g * g)")
            trng = np.random.default_rng(rank_seed(w, rank) + 77)
            table = torch.from_numpy((trng.standard_normal((H, binattn.relpos_table_entries(g, g, 0))) * 0.05)
                                     .astype(np.float32)).to(dev).bfloat16()
            rws = torch.empty(max(16, binattn.lib().binattn_forward_relpos_workspace_bytes(B, H, N, d)),
                              dtype=torch.uint8, device=dev)
            call = lambda: binattn.forward_relpos(qb, kb, aq, ak, table, (g, g), 0, v, scale, workspace=rws,
                                                  out=out, stream=stream)
        elif args.profile_path == "sample":
            if b is None:
                raise SystemExit("--profile-path sample needs the bias")
            sb = torch.cat([torch.roll(b, -i, dims=0).unsqueeze(0) for i in range(B)])
            sws = torch.empty(max(16, binattn.lib().binattn_forward_sample_bias_workspace_bytes(B, H, N, d, N)),
                              dtype=torch.uint8, device=dev)
            call = lambda: binattn.forward_sample_bias_ws(qb, kb, aq, ak, sb, v, scale, workspace=sws, out=out,
                                                          stream=stream)
        else:
            call = lambda: fwd(b)
        for _ in range(args.warmup):
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            call()
        torch.cuda.synchronize()
        binattn.device_status(stream)
        return

    # warm-up (untimed), including one checked run
    for _ in range(max(args.warmup, 3)):
        step(bias)
    binattn.device_status(stream)
    sampler = ClockSampler(local_rank)
    sampler.start()
    t_end = time.time() + 1.0
    while time.time() < t_end:  # clock soak, untimed
        for _ in range(20):
            flush.fill_(1)
            step(bias)
        torch.cuda.synchronize()

    results = {}
    for name, b in (("bias", bias), ("no_bias", None)):
        barrier()
        step_ms, fwd_ms = timed(b, args.steps)
        barrier()
        results[name] = dict(step_ms=max_over_ranks(sum(step_ms) / len(step_ms)),
                             fwd_ms=max_over_ranks(sum(fwd_ms) / len(fwd_ms)),
                             fwd_ms_median=statistics.median(fwd_ms),
                             fwd_ms_p10=percentile(fwd_ms, 0.1),
                             fwd_ms_p90=percentile(fwd_ms, 0.9),
                             fwd_ms_min=min(fwd_ms))
    clocks = sampler.stop()
    binattn.device_status(stream)

    # the same step with Q binarised inside the forward (binattn_forward_fused_ws):
    # pack(K) + the fused forward; its own timed region, same protocol
    fused = {}
    if args.engine == "auto":
        for name, b in (("bias", bias), ("no_bias", None)):
            need = binattn.fused_workspace_bytes(B, H, N, d, q.dtype, b is not None)
            fws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

            def fstep():
                binattn.pack(k, kb, ak, stream)
                binattn.forward_fused_ws(q, kb, ak, b, v, scale, workspace=fws, out=out, stream=stream)

            fstep()
            torch.cuda.synchronize()
            barrier()
            ev = []
            for _ in range(args.steps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fstep()
                e1.record(stream)
                ev.append((e0, e1))
            torch.cuda.synchronize()
            barrier()
            fused[name] = {"ms_per_step": round(max_over_ranks(sum(a.elapsed_time(c) for a, c in ev) / len(ev)), 5)}
            del fws
        binattn.device_status(stream)

    # the 8-bit P.V variant (binattn_forward_int8: V's 8-bit code, the row-max
    # pass and the 8-bit pass), same step and protocol
    int8 = {}
    if args.engine == "auto" and d % 8 == 0 and d <= 80:
        for name, b in (("bias", bias), ("no_bias", None)):
            iws = torch.empty(max(16, binattn.int8_workspace_bytes(B, H, N, d, b is not None)), dtype=torch.uint8,
                              device=dev)
            f8 = lambda b=b, iws=iws: binattn.forward_int8(qb, kb, aq, ak, b, v, scale, workspace=iws, out=out,
                                                           stream=stream)
            step(b)
            f8()
            torch.cuda.synchronize()
            barrier()
            ev = []
            for _ in range(args.steps):
                flush.fill_(1)
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                e0.record(stream)
                binattn.pack(q, qb, aq, stream)
                binattn.pack(k, kb, ak, stream)
                e1.record(stream)
                f8()
                e2.record(stream)
                ev.append((e0, e1, e2))
            torch.cuda.synchronize()
            barrier()
            int8[name] = {"ms_per_step": round(max_over_ranks(sum(a.elapsed_time(c) for a, _, c in ev) / len(ev)), 5),
                          "forward_ms": round(max_over_ranks(sum(b_.elapsed_time(c) for _, b_, c in ev) / len(ev)), 5)}
            del iws
        binattn.device_status(stream)

    # the position-sensitive bias: a relative-position table of the square
    # patch grid (DiT's latent patches; no class token) instead of the dense
    # [H, N, N] bias, same step and protocol
    relpos = {}
    g = int(round(math.sqrt(N)))
    if args.engine == "auto" and g * g == N and d % 8 == 0 and d <= 80:
        R = binattn.relpos_table_entries(g, g, 0)
        trng = np.random.default_rng(rank_seed(w, rank) + 77)
        table = torch.from_numpy((trng.standard_normal((H, R)) * 0.05).astype(np.float32)).to(dev).bfloat16()
        rws = torch.empty(max(16, binattn.lib().binattn_forward_relpos_workspace_bytes(B, H, N, d)),
                          dtype=torch.uint8, device=dev)
        fr = lambda: binattn.forward_relpos(qb, kb, aq, ak, table, (g, g), 0, v, scale, workspace=rws, out=out,
                                            stream=stream)
        fr()
        torch.cuda.synchronize()
        barrier()
        ev = []
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            e1.record(stream)
            fr()
            e2.record(stream)
            ev.append((e0, e1, e2))
        torch.cuda.synchronize()
        barrier()
        binattn.device_status(stream)
        rms = max_over_ranks(sum(b_.elapsed_time(c) for _, b_, c in ev) / len(ev))
        relpos = {"grid": [g, g], "table_entries_per_head": R,
                  "ms_per_step": round(max_over_ranks(sum(a.elapsed_time(c) for a, _, c in ev) / len(ev)), 5),
                  "forward_ms": round(rms, 5), "call": "binattn_forward_relpos",
                  "roofline": roofline_line(w, False, peaks, rms * 1e-3,
                                            torch.cuda.get_device_properties(dev).multi_processor_count)}
        del table, rws

    # the context-aware form of the bias: one dense bias per batch entry
    # (binattn_forward_sample_bias_ws), entry b the workload's bias with its
    # heads rotated by b; same step and protocol. B times the bias bytes.
    sample_bias = {}
    if args.engine == "auto" and d % 8 == 0 and d <= 80 and bias is not None:
        sb = torch.cat([torch.roll(bias, -i, dims=0).unsqueeze(0) for i in range(B)])
        sws = torch.empty(max(16, binattn.lib().binattn_forward_sample_bias_workspace_bytes(B, H, N, d, N)),
                          dtype=torch.uint8, device=dev)
        fs = lambda: binattn.forward_sample_bias_ws(qb, kb, aq, ak, sb, v, scale, workspace=sws, out=out,
                                                    stream=stream)
        fs()
        torch.cuda.synchronize()
        barrier()
        ev = []
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            binattn.pack(q, qb, aq, stream)
            binattn.pack(k, kb, ak, stream)
            e1.record(stream)
            fs()
            e2.record(stream)
            ev.append((e0, e1, e2))
        torch.cuda.synchronize()
        barrier()
        binattn.device_status(stream)
        sms = max_over_ranks(sum(b_.elapsed_time(c) for _, b_, c in ev) / len(ev))
        sample_bias = {"bias_shape": [B, H, N, N], "call": "binattn_forward_sample_bias_ws",
                       "ms_per_step": round(max_over_ranks(sum(a.elapsed_time(c) for a, _, c in ev) / len(ev)), 5),
                       "forward_ms": round(sms, 5),
                       "roofline": roofline_line(w, True, peaks, sms * 1e-3,
                                                 torch.cuda.get_device_properties(dev).multi_processor_count,
                                                 bias_per_sample=True)
                       | {"traffic": ncu_traffic(f"{w.name}/sample_bias"),
                          "algorithmic_bytes": algorithmic(w, True, bias_per_sample=True)["bytes"]}}
        del sb, sws

    # the backward (binattn_backward: dV, the gradients of the scaled binary
    # Q and K, and dbias summed over the batch) for an upstream gradient dO,
    # timed over a few calls with a cold L2
    backward = None
    try:
        grng = np.random.default_rng(rank_seed(w, rank) + 99)
        gO = torch.from_numpy(grng.standard_normal((B, H, N, d), dtype=np.float32)).to(dev).bfloat16()
        bws = torch.empty(max(16, binattn.lib().binattn_backward_workspace_bytes(B, H, N, d)), dtype=torch.uint8,
                          device=dev)
        fb = lambda: binattn.backward(qb, kb, aq, ak, bias, v, gO, scale, workspace=bws, stream=stream)
        fb()
        torch.cuda.synchronize()
        barrier()
        ev = []
        for _ in range(min(args.steps, 3)):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fb()
            e1.record(stream)
            ev.append((e0, e1))
        torch.cuda.synchronize()
        barrier()
        binattn.device_status(stream)
        bms = max_over_ranks(sum(a.elapsed_time(c) for a, c in ev) / len(ev))
        ab = algorithmic_backward(w)
        t_mem = ab["bytes"] / (peaks["hbm_gbs"] * 1e9)
        t_tensor = ab["pv_like_flops"] / (peaks["bf16_tflops"] * 1e12) + \
            ab["qk_ops"] / (E4M3_OVER_BF16 * peaks["bf16_tflops"] * 1e12)
        t_roof = max(t_mem, t_tensor)
        backward = {"call": "binattn_backward (CUDA cores: rows kernel, columns kernel)", "ms": round(bms, 4),
                    "calls_timed": len(ev), "algorithmic_bytes": ab["bytes"],
                    "roofline": {"bound": "hbm" if t_mem >= t_tensor else "tensor",
                                 "t_roof_us": round(t_roof * 1e6, 2), "t_mem_us": round(t_mem * 1e6, 2),
                                 "t_tensor_us": round(t_tensor * 1e6, 2), "frac": round(t_roof / (bms * 1e-3), 5)}}
        del gO, bws
    except Exception as exc:  # reported, not fatal: the forward's numbers stand on their own
        backward = {"unavailable": str(exc).splitlines()[0]}

    # in-build bf16 attention on the same shapes (speed reference), with the
    # binary forward's launch plan (binattn_ref_bf16_forward_ws: persistent
    # whole pairs, split tail) and, beside it, without the workspace
    ref = None
    try:
        rws = torch.empty(max(16, binattn.lib().binattn_ref_bf16_forward_workspace_bytes(B, H, N, d, 1)),
                          dtype=torch.uint8, device=dev)
        variants = (("ws", lambda: binattn.ref_bf16_forward_ws(q, k, bias, v, scale, workspace=rws, out=out,
                                                                stream=stream)),
                    ("plain", lambda: binattn.ref_bf16_forward(q, k, bias, v, scale, out=out, stream=stream)))
        ref_ms = {}
        for name, f in variants:
            f()
            torch.cuda.synchronize()
            ev = []
            for _ in range(args.steps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                f()
                e1.record(stream)
                ev.append((e0, e1))
            torch.cuda.synchronize()
            ref_ms[name] = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / len(ev))
        binattn.device_status(stream)
        ref = {"forward_ms": round(ref_ms["ws"], 5), "call": "binattn_ref_bf16_forward_ws",
               "without_split_ms": round(ref_ms["plain"], 5)}
        del rws
    except Exception as exc:  # not built for this engine/shape
        ref = {"unavailable": str(exc).splitlines()[0]}

    # end to end through the public API: pinned host inputs -> device -> result
    # back. The product call is HostPipeline.run, which overlaps the copies of
    # (b, head group) chunks with the computation of others; the same step
    # with the copies in series on one stream is reported beside it.
    from diffusion_transformers_b200.pipeline import HostPipeline
    h_q = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
    h_k = torch.from_numpy(inp["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
    h_v = torch.from_numpy(inp["v"].view(np.int16)).view(torch.bfloat16).pin_memory()
    h_o = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    pipe = HostPipeline(B, H, N, d, device=dev, has_bias=True)
    pipe.run(h_q, h_k, h_v, bias, scale, h_o, stream)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        pipe.run(h_q, h_k, h_v, bias, scale, h_o, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        q.copy_(h_q, non_blocking=True)
        k.copy_(h_k, non_blocking=True)
        v.copy_(h_v, non_blocking=True)
        step(bias)
        h_o.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    del pipe

    # the other workloads of the parity suite, timed the same way (forward with bias)
    others = [] if sharded else time_configs([n for n in WORKLOADS if n != w.name], args, rank, world, dev,
                                             stream, peaks, flush, max_over_ranks)

    if rank != 0:
        return
    a = algorithmic(w, True)
    a0 = algorithmic(w, False)
    fwd_s = results["bias"]["fwd_ms"] * 1e-3
    eff_tflops = a["eff_flops"] / fwd_s / 1e12
    fwd0_s = results["no_bias"]["fwd_ms"] * 1e-3
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    roof = roofline_line(w, True, peaks, fwd_s, n_sm)
    roof0 = roofline_line(w, False, peaks, fwd0_s, n_sm)
    line = {
        "metric": METRIC,
        "value": round(results["bias"]["step_ms"], 5),
        "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(results["bias"]["step_ms"], 5),
        "higher_is_better": False, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
        "dtype": "bf16", "dtype_detail": "1-bit Q/K scores (exact int), fp32 softmax, bf16 P.V, fp32 accumulate",
        "data": "synthetic",
        "config": workload_config(w_job, True) | {"engine": args.engine,
                                                  "parallelism": (f"heads sharded x{world} ({w.H} per rank, "
                                                                  "no data-path collective)") if sharded
                                                  else f"replicas x{world}",
                                              "call": "binattn_forward_ws" if ws["bias"] is not None
                                              else "binattn_forward"},
        "forward_ms": round(results["bias"]["fwd_ms"], 5),
        "forward_ms_median": round(results["bias"]["fwd_ms_median"], 5),
        "forward_ms_p10": round(results["bias"]["fwd_ms_p10"], 5),
        "forward_ms_p90": round(results["bias"]["fwd_ms_p90"], 5),
        "pack_ms": round(results["bias"]["step_ms"] - results["bias"]["fwd_ms"], 5),
        "effective_tflops": round(eff_tflops, 2),
        "job_effective_tflops": round((algorithmic(w_job, True)["eff_flops"] if sharded
                                       else job_units(a["eff_flops"], world)) / fwd_s / 1e12, 2),
        "fused_q_step": dict(fused, step="pack(K) + binattn_forward_fused_ws (Q binarised in the forward)"),
        "no_bias": {"ms_per_step": round(results["no_bias"]["step_ms"], 5),
                    "forward_ms": round(results["no_bias"]["fwd_ms"], 5),
                    "effective_tflops": round(a0["eff_flops"] / fwd0_s / 1e12, 2),
                    "roofline": roof0},
        "bf16_reference": ref,
        "relpos_bias": relpos,
        "per_sample_bias": sample_bias,
        "backward": backward,
        "int8_pv": dict(int8, call="binattn_forward_int8 (V 8-bit code + row-max pass + 8-bit P.V pass)",
                        step="pack(Q) + pack(K) + binattn_forward_int8"),
        "other_workloads": others,
        "roofline": roof | {
            "traffic": ncu_traffic(f"{w.name}/bias"),
            "traffic_unit": "bytes per forward call (its 3 launches)",
            "algorithmic_bytes": a["bytes"],
            "kernel": "binattn forward (with bias)",
            "peak_source": (peaks["source"] + " (burst): HBM copy GB/s; bf16 TFLOP/s for P.V, "
                            f"x{E4M3_OVER_BF16:g} for the e4m3 QK pipe (nominal 4.5/2.25 PFLOP/s)"),
            "t_exp_floor_basis": f"1 ex2 per pair at {MUFU_EXP_PER_CLK_PER_SM}/clk/SM, {n_sm} SMs, "
                                 f"{peaks.get('sm_max_mhz', 1965.0):g} MHz"},
        "e2e": {"value": round(e2e_ms, 4), "unit": "ms",
                "h2d_bytes_per_step": int(3 * B * H * N * d * 2),
                "d2h_bytes_per_step": int(B * H * N * d * 2),
                "call": "diffusion_transformers_b200.pipeline.HostPipeline.run (copies of (b, head group) chunks "
                        "overlapped with the packs and forwards of others)",
                "serial_ms": round(e2e_serial_ms, 4)},
        "gpu_launches": args.steps * (step_launches(w, True, args.engine) + step_launches(w, False, args.engine)),
        "gpu_launches_counts": "kernels of the timed headline steps (with and without the bias)",
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w, True, args.cpu_seconds, inp)
        line["cpu_oracle_workloads"] = cpu_oracle_all(w.name)
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        if not args.profile_once or args.batch < 1:
            raise SystemExit("--batch B (B >= 1) goes with --profile-once only")
        w = dataclasses.replace(w, B=args.batch)
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
