#!/usr/bin/env python
"""Benchmark of the Flint MoE-layer forward on B200 (one JSON line on stdout from rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode_int4] [--impl ours|reference]

A step is one forward of the whole layer (router -> top-k -> permutation -> experts -> combine) over
one batch of T synthetic tokens, inputs already resident in HBM. Between timed steps the L2 is
flushed by writing a 256 MiB buffer (outside the timed events). Steps are timed on the device with
CUDA events on the launching stream. With N > 1 (torchrun, one process per GPU) every rank runs its
own replica on its own batch (the layer is token-parallel; no collective is needed) and the time is
the max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this repository: there is no
reference implementation to install) on the host cores, on the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoE-layer tokens/s, HBM GB/s (% of 8 TB/s) at T=1..8; TFLOP/s % peak at T=2048"
H, I, IS = 2048, 512, 1024
HBM_NOMINAL_GBS = 8000.0
BF16_DENSE_NOMINAL_TFLOPS = 2250.0
FLUSH_BYTES = 256 << 20

WORKLOADS = {
    # name: (E, fmt, T, skew)
    "decode_int4": (256, "int4", 8, False),
    "prefill_int4": (256, "int4", 2048, False),
    "prefill_int4_skew": (256, "int4", 2048, True),
    "decode_nvfp4": (256, "nvfp4", 8, False),
    "prefill_nvfp4": (256, "nvfp4", 2048, False),
    "prefill_nvfp4_w4a4": (256, "nvfp4", 2048, False),
    "stack47_int4": (256, "int4", 8, False),
}
# stacks: layers of the workload (layer l drawn with seed 1000 + l); T tokens decode through all of them
STACK_LAYERS = {"stack47_int4": 47}
# W4A4: the routed experts' activations quantised to NVFP4, block-scaled FP4 MMAs
W4A4_WORKLOADS = {"prefill_nvfp4_w4a4"}
FP4_OVER_BF16_NOMINAL = 4.0          # dense FP4 / dense bf16 tensor rate (9 / 2.25 PFLOP/s)
# weight preparation: the bf16 gate|up and down banks of all E experts quantised once per step
QUANT_WORKLOADS = {"quant_int4": (256, "int4"), "quant_nvfp4": (256, "nvfp4")}
QUANT_SEED = 7
STACK_EPS = 1e-6


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="decode_int4", choices=sorted(WORKLOADS) + sorted(QUANT_WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-extras", action="store_true", help="skip the per-T decode and prefill side measurements")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the CPU-oracle baseline sample")
    p.add_argument("--quant-experts", type=int, default=0,
                   help="quant_* workloads: experts per step (default: all of the workload's); for small profiles")
    return p.parse_args()


# --------------------------------------------------------------------------------------------- workload math

def expert_bytes(fmt: str) -> int:
    if fmt == "int4":
        return 3 * H * I // 2 + (2 * I * (H // 128) + H * (I // 128)) * 2
    return 3 * H * I // 2 + 2 * I * (H // 16) + H * (I // 16) + 3 * 4


def algorithmic_bytes(E: int, fmt: str, T: int, n_active: int) -> int:
    """Bytes one forward must move at least: the touched experts, the shared expert, the router, x and y."""
    shared = (2 * IS * H + H * IS) * 2
    router = E * H * 2
    return n_active * expert_bytes(fmt) + shared + router + 2 * T * H * 2


def grouped_gemm_flops(T: int, K: int = 6) -> int:
    routed = 2 * T * K * (2 * I * H + H * I)
    shared = 2 * T * (2 * IS * H + H * IS)
    return routed + shared


def stage_bytes(name: str, E: int, fmt: str, T: int, K: int, n_active: int, w4a4: bool = False) -> int:
    """Algorithmic bytes of one kernel launch (weights it must stream plus its activations)."""
    P = T * K
    eb_gu = 2 * I * H // 2 + (2 * I * (H // 128) * 2 if fmt == "int4" else 2 * I * (H // 16) + 8)
    eb_dn = H * I // 2 + (H * (I // 128) * 2 if fmt == "int4" else H * (I // 16) + 4)
    sc_x = T * (H // 128) * 4 if fmt == "int4" else 0          # units of the 16-bit activation limbs
    sc_h = P * (I // 128) * 4 if fmt == "int4" else 0
    if w4a4:
        xa = P * (H // 2 + H // 16 + 4)                        # NVFP4 rows: codes, block scales, tensor scale
        ha = P * (I // 2 + I // 16 + 4)
        w4 = {"xq": T * H * 2 + xa + P * 4,
              "gu_routed": n_active * eb_gu + xa + P * I * 4,
              "hq": P * I * 4 + ha,
              "dn_routed": n_active * eb_dn + ha + P * H * 2}
        if name in w4:
            return w4[name]
    return {
        # decode path (T <= 8): one kernel moves the whole layer
        "layer": algorithmic_bytes(E, fmt, T, n_active),
        # larger T: one kernel per step (tensor-core path)
        "router_logits": E * H * 2 + T * H * 2 + T * E * 4,
        "topk": 4 * T * E * 4 + T * E * 4 + P * 8,              # 4 partial-logit slices in, logits out
        "permute": P * 4 * 3 + (E + 1) * 4,
        "xq": T * H * 2 + P * H * 2 + P * 4,
        "gu_routed": n_active * eb_gu + P * H * 2 + P * I * 2,
        "dn_routed": n_active * eb_dn + P * I * 2 + P * H * 2,
        "gu_shared": 2 * IS * H * 2 + T * H * 2 + T * IS * 4,
        "dn_shared": H * IS * 2 + T * IS * 4 + T * H * 4,
        "combine": P * H * 2 + T * H * 4 + T * H * 2 + P * 8,
    }.get(name, 0)


def stage_flops(name: str, E: int, T: int, K: int) -> int:
    """Multiply-add work (2 flops each) of one kernel launch of the tensor-core path."""
    P = T * K
    return {
        "router_logits": 2 * T * E * H,
        "gu_routed": 2 * P * 2 * I * H,
        "dn_routed": 2 * P * H * I,
        "gu_shared": 2 * T * 2 * IS * H,
        "dn_shared": 2 * T * H * IS * 2,      # bf16 pair (hi + lo) of the hidden activations
    }.get(name, 0)


def prefill_roofline(name: str, kernel_ms: float, E: int, fmt: str, T: int, n_active: int, peaks: dict,
                     workload: str, w4a4: bool) -> dict:
    """Roofline of one prefill kernel. W4A16: against the bf16 tensor peak (the kernel computes fp16,
    same rate). W4A4: the FP4 peak is the measured bf16 peak x the nominal FP4/bf16 ratio, and the
    kernel is judged against whichever of HBM and tensor time is the larger at its sizes."""
    st_flops = stage_flops(name, E, T, 6)
    st_bytes = stage_bytes(name, E, fmt, T, 6, n_active, w4a4)
    sec = kernel_ms * 1e-3
    tf = st_flops / sec / 1e12
    gbs = st_bytes / sec / 1e9
    base = {"kernel": name, "traffic": ncu_traffic(name, workload), "algorithmic_flops": st_flops,
            "algorithmic_bytes": st_bytes, "kernel_us": round(kernel_ms * 1e3, 2)}
    if not w4a4:
        return {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tf / peaks["bf16_tflops"], 4), "hbm_GB_per_s": round(gbs, 1), **base,
                "peak_source": peaks["source"] + " (bf16 burst; the kernel computes fp16 at the same rate)"}
    fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16_NOMINAL
    t_hbm, t_tc = st_bytes / (peaks["hbm_gbs"] * 1e9), st_flops / (fp4 * 1e12)
    if t_hbm >= t_tc:
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "tensor_TFLOPs": round(tf, 2), "fp4_peak_TFLOPs": round(fp4, 1),
                **base, "peak_source": peaks["source"] + " (burst copy; HBM time exceeds FP4 tensor time here)"}
    return {"bound": "tensor", "achieved": round(tf, 2), "peak": round(fp4, 1), "unit": "TFLOP/s",
            "frac": round(tf / fp4, 4), "hbm_GB_per_s": round(gbs, 1), **base,
            "peak_source": peaks["source"] + " (bf16 burst x 4, the nominal dense FP4/bf16 ratio)"}


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def ncu_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch of `kernel` from the committed ncu summary, if it was taken on
    the current kernel sources (source hash recorded beside the number); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = source_hash(traffic_sources(kernel, workload))
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        f = dict(kv.split("=", 1) for kv in line.split())
        if f.get("kernel") == kernel and f.get("workload") == workload and f.get("src") == cur:
            return int(float(f["dram_bytes_per_launch"]))
    return None


# the translation unit of each kernel whose DRAM traffic is recorded (profiles/ncu_traffic.txt): a
# recorded figure stands while these files are unchanged
TRAFFIC_SOURCES = {
    "layer": ("common.cuh", "decode.cu", "frag.cuh", "kernels.cuh"),
    "gu_routed": ("common.cuh", "kernels.cuh", "prefill.cu", "tc.cuh"),
    "quant": ("quant.cu",),
}
# W4A4 workloads: the routed kernels are those of w4a4.cu
TRAFFIC_SOURCES_W4A4 = {k: ("common.cuh", "kernels.cuh", "tc.cuh", "w4a4.cu") for k in ("gu_routed", "dn_routed")}


def traffic_sources(kernel: str, workload: str):
    if workload in W4A4_WORKLOADS and kernel in TRAFFIC_SOURCES_W4A4:
        return TRAFFIC_SOURCES_W4A4[kernel]
    return TRAFFIC_SOURCES.get(kernel)


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and with whitespace runs collapsed: what compiles."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash(files=None) -> str:
    """sha256 (first 12 hex digits) over the code of the named kernel sources (default: all of csrc), in
    name order; comments and layout do not count, so a figure survives edits that change no code."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_routed_expert_sigmoid_b200", "csrc")
    for fn in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:12]


# --------------------------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "50"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # nvidia-smi's start-up can hold driver locks for a while: wait for its first sample (up to 10 s)
        # so that it does not stall the launches of the timed region
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 10.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], None, set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# --------------------------------------------------------------------------------------------- ranks

def rank_first_row(rank: int, T: int) -> int:
    """Weak scaling: rank r decodes its own T token rows, [r*T, (r+1)*T) of the seeded stream."""
    return rank * T


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest of the ranks' values (every rank takes part; returns the input with one rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, T: int, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput: the tokens of every rank over the slowest rank's timed region."""
    return world * T * steps / (max_total_ms / 1e3)


# --------------------------------------------------------------------------------------------- ours

def measure_per_T(layer, fmt, E, Ts, redraws, timed_steps, steps, warmup, dev_name):
    """Decode forwards at each T: device time per forward and the HBM figures of its algorithmic bytes."""
    import torch

    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from bit_routed_expert_sigmoid_b200.layer import x_to_device
    out = {}
    for tt_ in Ts:
        xt = x_to_device(S.make_x(tt_, redraws=redraws), dev_name)
        yt = torch.empty((tt_, H), dtype=torch.bfloat16, device=dev_name)
        f = lambda: layer.forward(xt, yt)  # noqa: E731
        for _ in range(warmup):
            f()
        na = int((torch.diff(layer.routing(tt_)["offsets"]) > 0).sum().item())
        ms = statistics.mean(timed_steps(f, steps))
        ab = algorithmic_bytes(E, fmt, tt_, na)
        out[str(tt_)] = {"us": round(ms * 1e3, 2), "tokens_per_s": round(tt_ / (ms * 1e-3), 1),
                         "distinct_experts": na, "algorithmic_MB": round(ab / 1e6, 3),
                         "GB_per_s": round(ab / (ms * 1e-3) / 1e9, 1),
                         "pct_of_8TBps": round(100 * ab / (ms * 1e-3) / 1e9 / HBM_NOMINAL_GBS, 2)}
    return out


def measure_prefill(layer, fmt, E, skew, redraws, timed_steps, steps, dev_name, peaks, workload, w4a4=False):
    """One T = 2048 forward: device time, grouped-GEMM TFLOP/s, and the roofline of its slowest kernel
    (per-kernel CUDA-event times from the library's stage events, an instrumented pass that serialises
    the kernels)."""
    import torch

    from bit_routed_expert_sigmoid_b200 import binding as B
    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from bit_routed_expert_sigmoid_b200.layer import x_to_device
    Tp = 2048
    xp = x_to_device(S.make_x(Tp, redraws=redraws, skew=skew), dev_name)
    yp = torch.empty((Tp, H), dtype=torch.bfloat16, device=dev_name)
    f = lambda: layer.forward(xp, yp)  # noqa: E731
    for _ in range(3):
        f()
    ms = statistics.mean(timed_steps(f, steps))
    n_active = int((torch.diff(layer.routing(Tp)["offsets"]) > 0).sum().item())
    fl = grouped_gemm_flops(Tp)
    tf = fl / (ms * 1e-3) / 1e12
    stream = torch.cuda.current_stream()
    n_st = B.flint_moe_stage_count(layer.handle, Tp)
    names = [B.flint_moe_stage_name(layer.handle, Tp, i) for i in range(n_st)]
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    B.flint_moe_set_stage_events(layer.handle, [e.cuda_event for e in evs])
    acc = np.zeros(n_st)
    n_prof = max(3, steps // 2)
    for _ in range(n_prof):
        f()
        torch.cuda.synchronize()
        acc += [evs[i].elapsed_time(evs[i + 1]) for i in range(n_st)]
    B.flint_moe_set_stage_events(layer.handle, None)
    stage_ms = acc / n_prof
    top = int(np.argmax(stage_ms))
    return {"us": round(ms * 1e3, 1), "tokens_per_s": round(Tp / (ms * 1e-3), 1),
            "grouped_gemm_TFLOPs": round(tf, 2),
            "pct_of_2250TF_dense_bf16": round(100 * tf / BF16_DENSE_NOMINAL_TFLOPS, 2),
            "pct_of_measured_bf16": round(100 * tf / peaks["bf16_tflops"], 2),
            "distinct_experts": n_active,
            "stage_us_serialised": {n: round(float(t) * 1e3, 2) for n, t in zip(names, stage_ms)},
            "roofline": prefill_roofline(names[top], float(stage_ms[top]), E, fmt, Tp, n_active, peaks, workload,
                                         w4a4)}


def side_measurements(args, layer, redraws, timed_steps, dev_name, peaks) -> dict:
    """The other configurations of the layer, measured in the same run as the headline: NVFP4 decode
    (T = 1, 8), the T = 2048 prefill in both formats, with skewed expert loads (int4) and with NVFP4
    activations (W4A4)."""
    from bit_routed_expert_sigmoid_b200 import binding as B
    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer
    E = 256
    n_dec = min(args.steps, 1000)
    n_pf = max(3, min(args.steps // 20, 50))
    out = {"prefill_T2048": measure_prefill(layer, "int4", E, False, redraws, timed_steps, n_pf, dev_name, peaks,
                                            "prefill_int4")}
    Ls = S.make_layer(E, "int4", skew=True)
    lay = FlintMoELayer(Ls, t_max=2048, device=dev_name)
    del Ls
    out["prefill_T2048_skew"] = measure_prefill(lay, "int4", E, True, S.redraw_table(E, skew=True), timed_steps,
                                                n_pf, dev_name, peaks, "prefill_int4_skew")
    lay.close()
    Ln = S.make_layer(E, "nvfp4")
    lay = FlintMoELayer(Ln, t_max=2048, device=dev_name)
    out["per_T_nvfp4"] = measure_per_T(lay, "nvfp4", E, (1, 8), redraws, timed_steps, n_dec, args.warmup, dev_name)
    out["prefill_T2048_nvfp4"] = measure_prefill(lay, "nvfp4", E, False, redraws, timed_steps, n_pf, dev_name, peaks,
                                                 "prefill_nvfp4")
    lay.close()
    lay = FlintMoELayer(Ln, t_max=2048, device=dev_name, flags=B.FLINT_FLAG_W4A4)
    del Ln
    out["prefill_T2048_nvfp4_w4a4"] = measure_prefill(lay, "nvfp4", E, False, redraws, timed_steps, n_pf, dev_name,
                                                      peaks, "prefill_nvfp4_w4a4", w4a4=True)
    lay.close()
    return out


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch

    from bit_routed_expert_sigmoid_b200 import binding as B
    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer, x_to_device

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev_name = f"cuda:{local_rank}"
    torch.cuda.set_device(dev_name)
    E, fmt, T, skew = WORKLOADS[args.workload]
    K_TOP = 6
    L = S.make_layer(E, fmt, skew=skew)
    t_max = max(T, 8)
    w4a4 = args.workload in W4A4_WORKLOADS
    layer = FlintMoELayer(L, t_max=max(t_max, 2048 if not args.no_extras else t_max), device=dev_name,
                          flags=B.FLINT_FLAG_W4A4 if w4a4 else 0)
    # each rank takes its own batch of token rows (weak scaling: T tokens per GPU)
    redraws = S.redraw_table(E, skew=skew)
    x_bits = S.make_x(T, skew=skew, redraws=redraws, first_row=rank_first_row(rank, T))
    x = x_to_device(x_bits, dev_name)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev_name)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev_name)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def timed_steps(fn, K):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for i in range(K):
            flush.zero_()
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    fwd = lambda: layer.forward(x, y)  # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        fwd()
    n_active = int((torch.diff(layer.routing(T)["offsets"]) > 0).sum().item())

    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[0])
                          if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local_rank)
    clocks.start()
    barrier()
    wall0 = time.perf_counter()
    step_ms = timed_steps(fwd, args.steps)
    barrier()
    wall1 = time.perf_counter()
    total_ms = max_over_ranks(float(sum(step_ms)), dist, dev_name)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(world, T, args.steps, total_ms)

    # per-kernel times of the same forward (instrumented pass)
    n_st = B.flint_moe_stage_count(layer.handle, T)
    names = [B.flint_moe_stage_name(layer.handle, T, i) for i in range(n_st)]
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    B.flint_moe_set_stage_events(layer.handle, [e.cuda_event for e in evs])
    acc = np.zeros(n_st)
    n_prof = min(args.steps, 200)
    for _ in range(n_prof):
        flush.zero_()
        fwd()
        torch.cuda.synchronize()
        acc += [evs[i].elapsed_time(evs[i + 1]) for i in range(n_st)]
    B.flint_moe_set_stage_events(layer.handle, None)
    stage_ms = acc / n_prof
    top = int(np.argmax(stage_ms))
    peaks = measured_peaks()
    st_bytes = stage_bytes(names[top], E, fmt, T, K_TOP, n_active, w4a4)
    st_flops = stage_flops(names[top], E, T, K_TOP)
    if T > 8 and st_flops:
        roofline = prefill_roofline(names[top], float(stage_ms[top]), E, fmt, T, n_active, peaks, args.workload, w4a4)
    else:
        achieved = st_bytes / (stage_ms[top] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": names[top], "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": ncu_traffic(names[top], args.workload),
                    "algorithmic_bytes": st_bytes, "peak_source": peaks["source"] + " (burst copy)"}
    stages = {n: round(float(t) * 1e3, 2) for n, t in zip(names, stage_ms)}

    # end to end through the host-buffer entry point: H2D of x, forward, D2H of y
    xh = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
    yh = torch.empty((T, H), dtype=torch.int16).pin_memory()
    e2e_ms = timed_steps(lambda: layer.forward_host(xh, yh), min(args.steps, 500))
    e2e_total = float(sum(e2e_ms))
    if dist is not None:
        tt = torch.tensor([e2e_total], device=dev_name)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_total = float(tt.item())
    e2e = {"value": round(world * T * len(e2e_ms) / (e2e_total / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
           "ms_per_step": round(e2e_total / len(e2e_ms), 5)}

    extras = {}
    if not args.no_extras and world == 1 and args.workload == "decode_int4":
        extras["per_T"] = measure_per_T(layer, fmt, E, (1, 2, 4, 8), redraws, timed_steps, min(args.steps, 1000),
                                        args.warmup, dev_name)
    if not args.no_extras and world == 1 and args.workload == "decode_int4":
        extras.update(side_measurements(args, layer, redraws, timed_steps, dev_name, peaks))
    clk = clocks.stop()

    result = None
    if rank == 0:
        ab = algorithmic_bytes(E, fmt, T, n_active)
        cpu = cpu_baseline(args, L, x_bits, E) if world == 1 else None
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("w4a4: NVFP4 weights x NVFP4 activations (per-row fp32 scale, E4M3 per 16) on tcgen05 "
                      "kind::mxf4nvf4 block-scaled MMAs, fp32 accumulators in tensor memory; shared expert and "
                      "router bf16" if w4a4 else
                      "w4a16: int4 codes as exact int8 on the integer tensor cores against 16-bit fixed-point "
                      "activations (int32 sums), fp32 accumulate" if fmt == "int4" and T <= 8 else
                      "w4a16: fp16 tensor-core MMA, fp32 accumulate" if T <= 8 else
                      "w4a16: tcgen05 kind::f16 MMA (weights dequantised to exact fp16 in tensor memory, fp16 "
                      "activations), fp32 accumulators in tensor memory; shared expert and router bf16"),
            "data": "synthetic (seeded; random-init weights of the Flint MoE layer shape)",
            "config": {"workload": layer_workload(args.workload, E, fmt, T), "E": E, "T": T, "fmt": fmt,
                       "distinct_experts": n_active,
                       "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
                       "parallelism": f"replicas x{world} (token-parallel, no collective)"},
            "hbm": {"algorithmic_bytes": ab, "GB_per_s": round(ab / (ms_per_step * 1e-3) / 1e9, 1),
                    "pct_of_8TBps": round(100 * ab / (ms_per_step * 1e-3) / 1e9 / HBM_NOMINAL_GBS, 2),
                    "pct_of_measured": round(100 * ab / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 2)},
            "roofline": roofline, "stage_us": stages, "e2e": e2e,
            "gpu_launches": n_st * args.steps, "clocks": clk, "cpu_baseline": cpu,
            "wall_s_timed_region": round(wall1 - wall0, 4), **extras,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    layer.close()
    return result


# --------------------------------------------------------------------------------------------- CPU oracle

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(args, L, x_bits, E) -> dict:
    from oracle import flint_moe_ref as R
    T = x_bits.shape[0]
    Ts = min(T, 64)                      # bounded sample: the first 64 tokens of a larger batch
    xs = x_bits[:Ts]
    reps, t0 = 0, time.perf_counter()
    while True:
        R.moe_forward(L, xs, w4a4=args.workload in W4A4_WORKLOADS)
        reps += 1
        el = time.perf_counter() - t0
        if el >= args.cpu_seconds or reps >= 1000:
            break
    what = f"the same {T}-token batch" if Ts == T else f"the first {Ts} tokens of the {T}-token batch"
    return {"value": round(reps * Ts / el, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 oracle forward of {what}, repeated {reps}x in {el:.1f} s"}


def layer_workload(name: str, E: int, fmt: str, T: int) -> str:
    """config.workload of a one-layer workload: the same string on both arms."""
    return f"{name}: E={E} top-6, H=2048, I=512, shared 1024, {fmt}, T={T} tokens per GPU"


def stack_workload(name: str, n: int, E: int, fmt: str, T: int) -> str:
    return f"{name}: {n} layers x (E={E} top-6, H=2048, I=512, shared 1024, {fmt}), T={T}, x <- x + moe(rmsnorm(x))"


def quant_workload(name: str, E: int, fmt: str) -> str:
    return f"{name}: E={E} experts x (gate|up {2 * I}x{H}, down {H}x{I}) bf16 -> {fmt}"


def run_reference(args) -> dict:
    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from oracle import flint_moe_ref as R
    if args.workload in QUANT_WORKLOADS:
        E, fmt = QUANT_WORKLOADS[args.workload]
        bps, nbytes = quant_reference_sample(fmt, min(args.cpu_seconds, 30.0))
        v = round(bps / 1e9, 6)
        return {"impl": "reference", "metric": "weight preparation: bf16 GB/s quantised (all experts' gate|up "
                "and down banks)", "value": v, "unit": "GB/s", "n_gpus": 1, "steps": 1, "warmup": 0,
                "ms_per_step": round(nbytes / bps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32 decisions", "data": "synthetic",
                "config": {"workload": quant_workload(args.workload, E, fmt), "E": E, "fmt": fmt},
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"oracle quantiser on 64 rows x {H}, {nbytes / 1e6:.1f} MB"},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    E, fmt, T, skew = WORKLOADS[args.workload]
    if args.workload in STACK_LAYERS:
        # bounded sample: whole oracle stack steps on the first layers, the per-layer time scaled
        n = STACK_LAYERS[args.workload]
        x_bits = S.make_x(T, redraws=S.redraw_table(E))
        xs, times = R.bf16_to_f64(x_bits), []
        for l in range(max(1, min(args.steps, 3))):
            L = S.make_layer(E, fmt, seed=1000 + l)
            t1 = time.perf_counter()
            xs = R.stack_step(L, xs, eps=STACK_EPS)["x_next"]
            times.append(time.perf_counter() - t1)
        per_layer = float(np.mean(times))
        value = T / (per_layer * n)
        sample = f"fp64 oracle stack step on the first {len(times)} of {n} layers, per-layer time scaled to {n}"
        return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": 1,
                "steps": len(times), "warmup": 0, "ms_per_step": round(per_layer * n * 1e3, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": stack_workload(args.workload, n, E, fmt, T), "E": E,
                           "T": T, "fmt": fmt, "layers": n},
                "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": blas_threads(),
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    L = S.make_layer(E, fmt, skew=skew)
    # bounded sample: decode steps run whole; a prefill step runs the first 64 tokens of the batch
    Ts = T if T <= 64 else 64
    x_bits = S.make_x(Ts, skew=skew, redraws=S.redraw_table(E, skew=skew))
    for _ in range(min(args.warmup, 1)):
        R.moe_forward(L, x_bits, w4a4=args.workload in W4A4_WORKLOADS)
    steps = max(1, min(args.steps, 20 if Ts <= 8 else 5))
    t0 = time.perf_counter()
    for _ in range(steps):
        R.moe_forward(L, x_bits, w4a4=args.workload in W4A4_WORKLOADS)
    el = time.perf_counter() - t0
    value = steps * Ts / el
    cores = blas_threads()
    sample = f"fp64 oracle forward, {Ts} of the workload's {T} tokens per step, {steps} steps"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(el / steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": layer_workload(args.workload, E, fmt, T), "E": E, "T": T,
                       "fmt": fmt},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def quant_bytes_per_weight(fmt: str) -> float:
    """Algorithmic bytes per weight of the weight preparation: the bf16 read, the 4-bit code and the
    scale share (int4: a bf16 per 128; NVFP4: an E4M3 per 16, its amax pass re-reads the input)."""
    return 2.0 + 0.5 + (2.0 / 128 if fmt == "int4" else 1.0 / 16 + 2.0)


def quant_reference_sample(fmt: str, seconds: float):
    """The oracle quantiser on whole rows of one bank, for about `seconds`: bf16 bytes per second."""
    from oracle import quant_ref as Q
    rng = np.random.default_rng(QUANT_SEED)
    w = (rng.standard_normal((64, H)) * 0.02).astype(np.float32)
    wb = ((w.view(np.uint32).astype(np.uint64) + 0x7FFF + ((w.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16)
    done, t0 = 0, time.perf_counter()
    while True:
        if fmt == "int4":
            Q.quantize_int4_g128(wb, rotate=True)
        else:
            Q.quantize_nvfp4(wb)
        done += wb.nbytes
        if time.perf_counter() - t0 >= seconds:
            break
    return done / (time.perf_counter() - t0), done


def run_quant(args) -> dict:
    """Weight preparation of every expert of a layer: bf16 gate|up [E][2I][H] and down [E][H][I]
    (normal, std 0.02, drawn on the device from a seeded generator) into the layer's format."""
    import torch

    from bit_routed_expert_sigmoid_b200 import binding as B

    E, fmt = QUANT_WORKLOADS[args.workload]
    if args.quant_experts > 0:
        E = min(E, args.quant_experts)
    I = 512
    dev = "cuda:0"
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(QUANT_SEED)
    gu = (torch.randn((E, 2 * I, H), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    dn = (torch.randn((E, H, I), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    n_w = gu.numel() + dn.numel()
    if fmt == "int4":
        gc = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=dev)
        gs = torch.empty((E, 2 * I, H // 128), dtype=torch.int16, device=dev)
        dc = torch.empty((E, H, I // 2), dtype=torch.uint8, device=dev)
        ds = torch.empty((E, H, I // 128), dtype=torch.int16, device=dev)

        def step(w_gu=gu, w_dn=dn, e=E):
            B.flint_quantize_int4_g128(w_gu.data_ptr(), e * 2 * I, H, True, gc.data_ptr(), gs.data_ptr(), 0)
            B.flint_quantize_int4_g128(w_dn.data_ptr(), e * H, I, True, dc.data_ptr(), ds.data_ptr(), 0)
        launches = 2
    else:
        gc = torch.empty((2 * E, I, H // 2), dtype=torch.uint8, device=dev)
        gs = torch.empty((2 * E, I, H // 16), dtype=torch.uint8, device=dev)
        gt = torch.empty((2 * E,), dtype=torch.float32, device=dev)
        dc = torch.empty((E, H, I // 2), dtype=torch.uint8, device=dev)
        ds = torch.empty((E, H, I // 16), dtype=torch.uint8, device=dev)
        dt = torch.empty((E,), dtype=torch.float32, device=dev)

        def step(w_gu=gu, w_dn=dn, e=E):
            B.flint_quantize_nvfp4(w_gu.data_ptr(), 2 * e, I, H, gc.data_ptr(), gs.data_ptr(), gt.data_ptr(), 0)
            B.flint_quantize_nvfp4(w_dn.data_ptr(), e, H, I, dc.data_ptr(), ds.data_ptr(), dt.data_ptr(), 0)
        launches = 6
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms_per_step = float(np.mean(ms))
    in_bytes = 2 * n_w
    value = in_bytes / (ms_per_step * 1e-3) / 1e9
    peaks = measured_peaks()
    ab = quant_bytes_per_weight(fmt) * n_w
    achieved = ab / (ms_per_step * 1e-3) / 1e9
    kern = "quant_int4_kernel" if fmt == "int4" else "quant_amax_kernel + quant_nvfp4_kernel"
    roofline = {"bound": "hbm", "kernel": kern, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": ncu_traffic("quant", args.workload),
                "algorithmic_bytes": int(ab), "peak_source": peaks["source"] + " (burst copy)"}

    # end to end through the public API on a 16-expert slice: pinned host bf16 in, codes and scales out
    Ee = min(16, E)
    h_gu = gu[:Ee].cpu().pin_memory()
    h_dn = dn[:Ee].cpu().pin_memory()
    d_gu, d_dn = torch.empty_like(gu[:Ee]), torch.empty_like(dn[:Ee])
    outs = [t[: (2 * Ee if (fmt == "nvfp4" and t is gc) else Ee)] for t in (gc, dc)]
    h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

    def e2e_step():
        d_gu.copy_(h_gu, non_blocking=True)
        d_dn.copy_(h_dn, non_blocking=True)
        step(d_gu, d_dn, Ee)
        for o, ho in zip(outs, h_out):
            ho.copy_(o, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    k = max(3, min(args.steps, 20))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(k):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / k
    e_in = 2 * (h_gu.numel() + h_dn.numel())
    e2e = {"value": round(e_in / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": int(e_in),
           "d2h_bytes_per_step": int(sum(o.numel() * o.element_size() for o in outs)),
           "ms_per_step": round(e2e_ms, 4), "slice": f"{Ee} of the {E} experts (codes read back, scales not)"}
    clk = clocks.stop()
    cpu_bps, cpu_bytes = quant_reference_sample(fmt, args.cpu_seconds)
    return {
        "metric": "weight preparation: bf16 GB/s quantised (all experts' gate|up and down banks)",
        "value": round(value, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 decisions (IEEE, fixed order) from bf16 input" + (", 128-wide Hadamard rotation" if fmt == "int4" else ""),
        "data": "synthetic (seeded normal bf16 weights, std 0.02, drawn on the device)",
        "config": {"workload": quant_workload(args.workload, E, fmt),
                   "E": E, "fmt": fmt, "weights": int(n_w),
                   "l2": f"not flushed: {in_bytes / 1e9:.2f} GB of input per step, larger than the 126 MB L2",
                   "parallelism": "single GPU"},
        "roofline": roofline, "e2e": e2e, "gpu_launches": launches * args.steps, "clocks": clk,
        "cpu_baseline": {"value": round(cpu_bps / 1e9, 6), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"fp32-decision oracle quantiser on 64 rows x {H} bf16, {cpu_bytes / 1e6:.1f} MB "
                                   f"in {args.cpu_seconds:.0f} s"},
        "wall_s_timed_region": round(wall1 - wall0, 4),
    }


def run_stack(args) -> dict:
    """Decode of T tokens through a stack of independent seeded layers on the fp32 residual stream
    (z = bf16(rmsnorm(x)); x += layer(z)); the weights (20 GB at 47 layers) never stay in L2."""
    import torch

    from bit_routed_expert_sigmoid_b200 import binding as B
    from bit_routed_expert_sigmoid_b200 import synthetic as S
    from bit_routed_expert_sigmoid_b200.layer import FlintMoEStack

    E, fmt, T, skew = WORKLOADS[args.workload]
    n = STACK_LAYERS[args.workload]
    dev = "cuda:0"
    torch.cuda.set_device(dev)
    stack = FlintMoEStack((S.make_layer(E, fmt, seed=1000 + l) for l in range(n)), t_max=T, eps=STACK_EPS,
                          device=dev)
    x_bits = S.make_x(T, redraws=S.redraw_table(E))
    x0 = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).float().to(dev)     # residual = input
    x = x0.clone()
    stream = torch.cuda.current_stream()

    def timed_steps(fn, K):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for i in range(K):
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    fwd = lambda: stack.forward(x)  # noqa: E731
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    n_active = [int((torch.diff(layer.routing(T)["offsets"]) > 0).sum().item()) for layer in stack.layers]
    clocks = ClockSampler(0)
    clocks.start()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    step_ms = timed_steps(fwd, args.steps)
    wall1 = time.perf_counter()
    total_ms = float(sum(step_ms))
    ms_per_step = total_ms / args.steps
    value = T * args.steps / (total_ms / 1e3)
    glue = (n + 1) * T * H * (4 + 4 + 2 + 2)          # residual read + write, y read, z write per boundary
    ab = sum(algorithmic_bytes(E, fmt, T, a) for a in n_active) + glue

    # the layer kernel of every layer, timed with the library's stage events (instrumented pass)
    n_st = B.flint_moe_stage_count(stack.layers[0].handle, T)
    names = [B.flint_moe_stage_name(stack.layers[0].handle, T, i) for i in range(n_st)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)] for _ in stack.layers]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for layer, row in zip(stack.layers, evs):
        B.flint_moe_set_stage_events(layer.handle, [e.cuda_event for e in row])
    acc = np.zeros((n, n_st))
    n_prof = max(1, min(args.steps, 20))
    for _ in range(n_prof):
        fwd()
        torch.cuda.synchronize()
        acc += [[row[i].elapsed_time(row[i + 1]) for i in range(n_st)] for row in evs]
    for layer in stack.layers:
        B.flint_moe_set_stage_events(layer.handle, None)
    stage_ms = acc / n_prof
    gi = names.index("layer")
    gu_bytes = sum(stage_bytes("layer", E, fmt, T, 6, a) for a in n_active)
    gu_ms = float(stage_ms[:, gi].sum())
    peaks = measured_peaks()
    achieved = gu_bytes / (gu_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "layer (every layer)", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": None, "algorithmic_bytes": gu_bytes, "peak_source": peaks["source"] + " (burst copy)"}

    # end to end through the public API: H2D of the residual, the stack, D2H of the residual
    xh = torch.empty((T, H), dtype=torch.float32).pin_memory()
    xh.copy_(x0.cpu())

    def e2e_step():
        x.copy_(xh, non_blocking=True)
        stack.forward(x)
        xh.copy_(x, non_blocking=True)
    e2e_ms = timed_steps(e2e_step, min(args.steps, 200))
    e2e = {"value": round(T * len(e2e_ms) / (sum(e2e_ms) / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4,
           "ms_per_step": round(float(sum(e2e_ms)) / len(e2e_ms), 5)}
    clk = clocks.stop()
    errors = [layer.error_word() for layer in stack.layers]

    # bounded CPU baseline (the oracle leg): the oracle on the first layers, per-layer time scaled
    from oracle import flint_moe_ref as R
    t0 = time.perf_counter()
    done, xs = 0, R.bf16_to_f64(x_bits)
    while done < n:
        L = S.make_layer(E, fmt, seed=1000 + done)
        t1 = time.perf_counter()
        xs = R.stack_step(L, xs, eps=STACK_EPS)["x_next"]
        el_layer = time.perf_counter() - t1
        done += 1
        if time.perf_counter() - t0 >= args.cpu_seconds:
            break
    cpu_layer_s = el_layer
    cpu = {"value": round(T / (cpu_layer_s * n), 4), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"fp64 oracle stack step on {done} of the {n} layers ({cpu_layer_s:.2f} s for the last), "
                     f"scaled to {n} layers"}
    stack.close()
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "w4a16: int4 codes as exact int8 on the integer tensor cores against 16-bit fixed-point "
                 "activations (int32 sums), fp32 accumulate; fp32 residual stream",
        "data": "synthetic (seeded; random-init weights of the Flint MoE layer shape, layer l seed 1000+l)",
        "config": {"workload": stack_workload(args.workload, n, E, fmt, T), "E": E, "T": T, "fmt": fmt, "layers": n,
                   "distinct_experts_per_layer": round(float(np.mean(n_active)), 2),
                   "l2": f"not flushed: {stack.weight_bytes() / 1e9:.1f} GB of weights stream through the 126 MB L2",
                   "parallelism": "single GPU"},
        "hbm": {"algorithmic_bytes": ab, "GB_per_s": round(ab / (ms_per_step * 1e-3) / 1e9, 1),
                "pct_of_8TBps": round(100 * ab / (ms_per_step * 1e-3) / 1e9 / HBM_NOMINAL_GBS, 2),
                "pct_of_measured": round(100 * ab / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 2)},
        "per_layer_us": round(ms_per_step * 1e3 / n, 2),
        "roofline": roofline,
        "stage_us_per_layer": {nm: round(float(stage_ms[:, i].mean()) * 1e3, 2) for i, nm in enumerate(names)},
        "e2e": e2e, "gpu_launches": (n * (n_st + 1) + 1) * args.steps, "clocks": clk, "cpu_baseline": cpu,
        "error_words": sorted(set(errors)), "wall_s_timed_region": round(wall1 - wall0, 4),
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.workload in STACK_LAYERS:
        if rank == 0:
            print(json.dumps(run_stack(args)), flush=True)
        return
    if args.workload in QUANT_WORKLOADS:
        if rank == 0:
            print(json.dumps(run_quant(args)), flush=True)
        return
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
