#!/usr/bin/env python3
"""Throughput of the routed-expert MoE layer on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one pass of the whole hot path over one batch of synthetic tokens:
router GEMM + softmax/top-k + renormalisation, permutation by expert, grouped
SwiGLU experts (gate/up + SwiGLU, down), the shared expert, and the weighted
combine (the Refill workload adds the Refill-RMS accumulation and the
selection).  The default workload is the BF16 layer at Flash-Next shape in
prefill: T=8192 tokens, H=2048, E=512 experts, top-10, expert width 640, one
shared expert of width 640.

`value` is whole-job tokens/s (tokens of all ranks / the slowest rank's
time), timed with CUDA events on the launching stream over exactly K steps
with inputs resident in HBM.  `e2e` repeats the measurement through the same
public API with the token batch copied from pinned host memory and the layer
output copied back inside every step.  Under torchrun every rank runs its own
batch (weak scaling; the forward has no collective).

--impl reference times the CPU oracle (oracle/, float64 NumPy) on a bounded
sample of the same workload on this machine's host cores.
"""

from __future__ import annotations

import argparse
import dataclasses
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_expert_gemm_b200 import MoELayer, abi, synth  # noqa: E402
from bit_expert_gemm_b200.layer import HostPipeline, slice_layer_weights  # noqa: E402

METRIC = "MoE-layer tokens/s at E=512,k=10 (prefill TFLOP/s & decode HBM GB/s vs roofline)"
L2_BYTES = 126 * 1024 * 1024
# denominators when MEASURED_PEAKS.json is absent, and the nominal B200 figures
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_HBM_GBS = 8000.0
# decode rows measured beside the default prefill line (the metric's decode half)
DECODE_COMPANIONS = ("bf16_decode_t1", "bf16_decode_t64")

# name -> (synth workload, T, kind)
WORKLOADS = {
    "bf16_prefill": ("bf16", 8192, "forward"),
    "bf16_decode_t1": ("bf16", 1, "forward"),
    "bf16_decode_t8": ("bf16", 8, "forward"),
    "bf16_decode_t64": ("bf16", 64, "forward"),
    "awq_prefill": ("awq_g32", 8192, "forward"),
    "awq_decode_t1": ("awq_g32", 1, "forward"),
    "awq_decode_t8": ("awq_g32", 8, "forward"),
    "awq_decode_t32": ("awq_g32", 32, "forward"),
    # the AWQ card's BF16 mode (BF16 activations, scales rounded to BF16)
    "awq_bf16_prefill": ("awq_g32_bf16", 8192, "forward"),
    "awq_bf16_decode_t1": ("awq_g32_bf16", 1, "forward"),
    "nvfp4_prefill": ("nvfp4", 16384, "forward"),
    "nvfp4_decode_t1": ("nvfp4", 1, "forward"),
    "nvfp4_decode_t8": ("nvfp4", 8, "forward"),
    "nvfp4_decode_t64": ("nvfp4", 64, "forward"),
    "bf16_h2560_prefill": ("bf16_h2560", 8192, "forward"),
    # small case of the same kernels for full ncu captures (64 experts, 2048 tokens)
    "profile_e64_t2048": ("profile_e64", 2048, "forward"),
    "refill": ("refill", 32768, "refill"),
    # RAZOR-pruned layers (the 65B and 96B budgets): the E=512 BF16 layer's
    # Refill-RMS statistics over one 32768-token calibration row, the top 256
    # or 384 experts kept, router rows, bias and expert weights sliced on the
    # device, then the forward of the pruned layer
    "bf16_razor256_prefill": ("bf16", 8192, "forward"),
    "bf16_razor384_prefill": ("bf16", 8192, "forward"),
    "bf16_razor256_decode_t1": ("bf16", 1, "forward"),
    # the BF16 layer with its pre-MoE RMSNorm (gain 1 + w, eps 1e-6) and a
    # shared-expert gate, both inside the routing call
    "bf16_norm_prefill": ("bf16", 8192, "forward"),
    "bf16_norm_decode_t1": ("bf16", 1, "forward"),
}
PRUNED = {"bf16_razor256_prefill": 256, "bf16_razor384_prefill": 384, "bf16_razor256_decode_t1": 256}
WITH_NORM = {"bf16_norm_prefill", "bf16_norm_decode_t1"}
CALIBRATION_T = 32768


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="bf16_prefill", choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="launch the C-ABI calls eagerly instead of a CUDA graph")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true",
                   help="skip the decode rows (T=1, T=64) that the default prefill line carries")
    p.add_argument("--cpu-sample-tokens", type=int, default=0, help="oracle sample size (0: automatic)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no collective in the data path)
# ---------------------------------------------------------------------------
class Dist:
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE): NCCL
    for the barrier and the max over ranks of the device-timed region; gloo
    on hosts without CUDA (the CPU tests of this logic)."""

    def __init__(self, backend: str = ""):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=300), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """Polls the SM clock and the clock-event (throttle) reasons through NVML
    every 2 ms while the timed region runs."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int):
        self.sm, self.mx, self.bits = [], [], 0
        self.err = None
        self.stop_flag = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.get_reasons = get
            self.mx.append(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception as e:  # no NVML: report it instead of a number
            self.err = f"NVML unavailable: {e}"

    def _sample(self):
        self.sm.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        self.bits |= int(self.get_reasons(self.h))

    def _run(self):
        while not self.stop_flag.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self) -> dict:
        if self.err:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err]}
        self.stop_flag.set()
        self.t.join(timeout=1)
        self._sample()
        reasons = sorted(n for n, b in self.REASONS.items() if self.bits & b)
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": max(self.mx), "reasons": reasons,
                "samples": len(self.sm)}


BAD_CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clk: dict) -> bool:
    """True when a timed region's clock record does not stand: a hardware or
    thermal slowdown was active, or the SM clock stayed well below its
    maximum with no reason reported (a clock lock left on the GPU).  A power
    cap alone is normal for a dense GEMM on this part and is kept."""
    if clk.get("sm_mhz") is None or not clk.get("sm_max_mhz"):
        return False  # no NVML record: nothing to judge
    if any(r in BAD_CLOCK_REASONS for r in clk["reasons"]):
        return True
    return not clk["reasons"] and clk["sm_mhz"] < 0.85 * clk["sm_max_mhz"]


def measured_peaks() -> dict:
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {}


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; also the --impl reference arm)
# ---------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# tokens per oracle call, for the cpu_baseline leg and each reference-arm step:
# large enough that the per-call conversion of the touched experts' weights
# to float64 is a small part of a call
CPU_SAMPLE_TOKENS = {"forward": 1024, "refill": 512}


def oracle_tokens_per_s(wl, w, x: torch.Tensor, n_tokens: int, kind: str):
    """Runs the float64 oracle on the first n_tokens tokens; returns (tokens/s, seconds)."""
    from oracle import awq, moe, nvfp4, razor

    I = wl.I

    def to64(t):
        return t.detach().float().cpu().double().numpy()

    cache = {}
    if wl.fmt == "awq_g32":
        host = {k: w[k].cpu().numpy() for k in EXPERT_KEYS["awq_g32"]}

    def ew(e):
        if e not in cache:
            if wl.fmt == "awq_g32":
                cache[e] = awq.expert_weights_out_in(host["qw_gu"], host["qz_gu"], host["sc_gu"], host["qw_d"],
                                                     host["qz_d"], host["sc_d"], e, I,
                                                     mode="bf16" if wl.act == "bf16" else "fp16")
            else:
                g = to64(w["w_gate_up"][e])
                ws = (g[:I], g[I:], to64(w["w_down"][e]))
                if wl.fmt == "nvfp4":
                    ws = tuple(nvfp4.fake_quant(m.astype(np.float32)) for m in ws)
                cache[e] = ws
        return cache[e]

    xs = to64(x[:n_tokens])
    wr, b = to64(w["w_router"]), to64(w["bias"])
    sh = to64(w["w_sh_gate_up"])
    shared = (sh[: wl.I_sh], sh[wl.I_sh:], to64(w["w_sh_down"]))
    gate_w = to64(w["w_sh_gate"]) if "w_sh_gate" in w else None
    t0 = time.perf_counter()
    if "w_norm" in w:
        xs = moe.block_input(xs, to64(w["w_norm"]), 1e-6, dtype="bf16" if wl.act == "bf16" else "f16")
    if kind == "refill":
        out = moe.moe_layer(xs, wr, b, wl.k, ew, shared, extra=1)
        r = out["route"]
        d = razor.refill_deltas_closed_form(out["f"], out["perm"]["slot_row"], r["idx"], r["p"], wl.k)
        s, c = np.zeros(wl.E), np.zeros(wl.E, np.int64)
        razor.accumulate(s, c, d, r["idx"], wl.k)
        razor.select(s, c, wl.keep)
    elif wl.fmt == "nvfp4":
        r = moe.route(xs, wr, b, wl.k)
        perm = moe.permute(r["idx"], wl.E)
        f, _, _ = nvfp4.routed_outputs_w4a4(xs, perm, ew)
        moe.combine(f, perm["slot_row"], r["w"], moe.swiglu_expert(xs, *shared)[0])
    else:
        moe.moe_layer(xs, wr, b, wl.k, ew, shared, shared_gate_w=gate_w)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


# ---------------------------------------------------------------------------
def expert_flops(rows: int, H: int, I: int) -> float:
    return 2.0 * rows * 3 * H * I


EXPERT_KEYS = {"bf16": ("w_gate_up", "w_down"), "awq_g32": ("qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d"),
               "nvfp4": ("w_gu", "sf_gu", "gs_gu", "w_d", "sf_d", "gs_d")}
KERNEL_NAMES = {"bf16": "moe_experts_bf16 (routed + shared experts: GEMM1/SwiGLU + GEMM2, tcgen05 kind::f16; "
                        "decode-sized batches stream the weights as the M operand)",
                "awq_g32": "moe_experts_awq_g32_prepacked (routed AWQ experts from the tile-packed copy: "
                           "dequantising GEMM1/SwiGLU gathering its x rows + dequantising GEMM2, tcgen05 kind::f16; "
                           "T <= 16: the split-K weight-streaming kernel; + the FP16 shared expert)",
                "nvfp4": "moe_grouped_swiglu_nvfp4_prepacked (activation quantisation + GEMM1/SwiGLU + h "
                         "quantisation + GEMM2: tcgen05 kind::mxf4nvf4; T <= 16: CUDA-core GEMVs with exact dp4a "
                         "group products) + the BF16 shared expert (T <= 16: weight-streaming GEMVs on a second "
                         "stream)"}


def measured_traffic(workload: str):
    """DRAM bytes per expert call from the committed ncu summaries under
    profiles/: a line `traffic: workload=W bytes_per_launch=N sources=a,b
    sha256=H`.  The hash is over the listed kernel sources as they were when
    the counters were taken; if the sources have changed since, the figure no
    longer belongs to the kernel that runs and None is returned."""
    pat = re.compile(r"traffic: workload=(\S+) bytes_per_launch=(\d+) sources=(\S+) sha256=([0-9a-f]+)")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(path):
            m = pat.search(line)
            if not m or m.group(1) != workload:
                continue
            h = hashlib.sha256()
            try:
                for f in m.group(3).split(","):
                    with open(os.path.join(ROOT, "bit_expert_gemm_b200", "csrc", f), "rb") as fh:
                        h.update(fh.read())
            except OSError:
                return None, None
            if h.hexdigest()[:len(m.group(4))] != m.group(4):
                return None, os.path.relpath(path, ROOT) + " (kernel sources changed since the capture)"
            return int(m.group(2)), os.path.relpath(path, ROOT)
    return None, None


def _count_step_kernels(layer, x, step) -> int:
    layer.capture(x, step, warmup=0)
    return layer.graph_kernels


def expert_roofline(wl, layers, T, rows, ffn_ms, peaks) -> dict:
    """Roofline of the routed expert call: tensor-bound (algorithmic FLOPs)
    for prefill-sized batches, HBM-bound (bytes of the distinct experts the
    batch touches, averaged over the timed units' last routings) for
    decode-sized ones."""
    layer = layers[0]
    w = layer.w
    keys = EXPERT_KEYS[wl.fmt]
    per_expert = sum(w[k].numel() * w[k].element_size() for k in keys) / wl.E
    touched_each = [int((torch.diff(lay.offsets.to(torch.int64)).cpu() > 0).sum()) for lay in layers]
    touched = statistics.mean(touched_each)
    expert_bytes = touched * per_expert
    flops = expert_flops(rows, wl.H, wl.I)
    with_shared = True  # the timed region (experts_and_shared) also runs the shared expert
    if with_shared:
        sh_bytes = sum(w[k].numel() * w[k].element_size() for k in ("w_sh_gate_up", "w_sh_down"))
        expert_bytes += sh_bytes
        flops += expert_flops(T, wl.H, wl.I_sh)
    if T >= 256:
        # the expert call is timed in runs of a few tens of milliseconds at full
        # clocks: a burst, so the burst cuBLAS figure is the denominator; the
        # sustained (power-capped, seconds-long) figure is reported beside it
        burst = peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)
        sustained = peaks.get("bf16_tflops_sustained")
        if wl.fmt == "nvfp4":
            peak = 4.0 * burst
            src = ("derived: 4 x the measured burst BF16 GEMM rate (MEASURED_PEAKS.json bf16_tflops) x the nominal "
                   "FP4:BF16 ratio 9/2.25; no FP4 peak is measured")
            nominal = NOMINAL_FP4_TFLOPS
        else:
            peak = burst
            src = ("measured burst (MEASURED_PEAKS.json bf16_tflops: cuBLAS bf16 8192^3, best of 10; the expert call "
                   "is timed the same way, in short runs at full clocks; FP16 runs at the BF16 rate)"
                   if "bf16_tflops" in peaks else "fallback 1590 TFLOP/s (no MEASURED_PEAKS.json)")
            nominal = NOMINAL_BF16_TFLOPS
        achieved = flops / (ffn_ms / 1e3) / 1e12
        out = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
               "frac": round(achieved / peak, 4), "traffic": None, "kernel": KERNEL_NAMES[wl.fmt],
               "work_per_launch": f"{flops / 1e9:.1f} GFLOP = 2*rows*3*H*I, rows={rows}"
                                  + (f" + shared expert on {T} tokens" if with_shared else ""), "peak_source": src,
               "frac_of_nominal": round(achieved / nominal, 4), "nominal_peak": nominal,
               "experts_touched": touched}
        if sustained and wl.fmt != "nvfp4":
            out["frac_of_sustained"] = round(achieved / sustained, 4)
        return out
    peak = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
    achieved = expert_bytes / (ffn_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": None, "kernel": KERNEL_NAMES[wl.fmt],
            "work_per_launch": f"{expert_bytes / 1e6:.2f} MB = {touched:.1f} experts x {per_expert / 1e6:.3f} MB"
                               + (" + the shared expert" if with_shared else ""),
            "peak_source": ("measured (MEASURED_PEAKS.json hbm_gbs: torch copy)" if "hbm_gbs" in peaks else
                            "fallback 6650 GB/s (no MEASURED_PEAKS.json)"),
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4), "nominal_peak": NOMINAL_HBM_GBS,
            "experts_touched": touched}


def razor_pruned_weights(wl, seed: int, keep: int, dev) -> dict:
    """The layer of seed `seed` pruned to `keep` experts the RAZOR way, all on
    the device through the C ABI: Refill-RMS statistics over one calibration
    row of CALIBRATION_T tokens, razor_select, razor_slice of every
    per-expert tensor with the kept set."""
    w = synth.make_weights(wl, seed=seed, device=dev)
    cal = MoELayer(w, wl.k, wl.fmt, T_max=CALIBRATION_T, extra=1)
    ss = torch.zeros(wl.E, dtype=torch.float64, device=dev)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=dev)
    cal.refill_pass(synth.make_tokens(wl, CALIBRATION_T, seed=seed, batch=1000, device=dev), ss, cc)
    kept, _, _ = abi.razor_select(ss, cc, keep)
    pruned = slice_layer_weights(w, kept)
    torch.cuda.synchronize()
    del cal, w
    torch.cuda.empty_cache()
    return pruned


def bench_workload(args, dist: Dist, workload: str, with_e2e: bool = True, with_cpu: bool = True) -> dict:
    """Measures one workload; returns its JSON line (not printed)."""
    wname, T, kind = WORKLOADS[workload]
    wl = synth.WORKLOADS[wname]
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    extra = 1 if kind == "refill" else 0
    decode = T < 256
    keep = PRUNED.get(workload, 0)
    if keep:
        wl_full = wl
        wl = dataclasses.replace(wl, E=keep)

        def layer_weights(seed):
            return razor_pruned_weights(wl_full, seed, keep, dev)
    elif workload in WITH_NORM:
        def layer_weights(seed):
            w = synth.make_weights(wl, seed=seed, device=dev)
            w["w_norm"] = synth.make_norm_weight(wl, seed, device=dev)
            w["w_sh_gate"] = synth.make_shared_gate(wl, seed, device=dev)
            return w
    else:
        def layer_weights(seed):
            return synth.make_weights(wl, seed=seed, device=dev)
    layers = [MoELayer(layer_weights(0), wl.k, wl.fmt, T_max=T, extra=extra)]
    layer_bytes = sum(t.numel() * t.element_size() for t in layers[0].w.values())
    if decode:
        # A decode step touches fewer expert bytes than L2 holds.  Rotate
        # through layers with distinct weights so that, between two uses of
        # one layer, the others stream at least 3x L2 of expert weights (at
        # least k routed experts + the shared expert per step): no expert
        # weight is L2-resident when its layer runs again.
        per_expert = sum(layers[0].w[k].numel() * layers[0].w[k].element_size() for k in EXPERT_KEYS[wl.fmt]) / wl.E
        step_min = (wl.k + 1) * per_expert
        n_layers = max(2, 1 + -(-3 * L2_BYTES // int(step_min)))
        n_layers = min(n_layers, 24, max(2, int(64e9 // layer_bytes)))
        for l in range(1, n_layers):
            layers.append(MoELayer(layer_weights(l), wl.k, wl.fmt, T_max=T, extra=extra))
    layer = layers[0]
    w = layer.w
    # token batches: distinct per rank, rotated so that the inputs of the
    # timed steps exceed the L2 cache
    x_bytes = T * wl.H * 2
    n_batches = max(2, min(8, -(-2 * L2_BYTES // x_bytes)))
    xs = [synth.make_tokens(wl, T, seed=1 + dist.rank, batch=b, device=dev) for b in range(n_batches)]
    # units of the rotation: (layer, token batch); one CUDA graph each
    units = ([(layers[l], xs[l % n_batches]) for l in range(len(layers))] if decode else
             [(layer, xs[b]) for b in range(n_batches)])
    n_units = len(units)
    sum_sq = torch.zeros(wl.E, dtype=torch.float64, device=dev)
    count = torch.zeros(wl.E, dtype=torch.int64, device=dev)
    kept = torch.empty(max(wl.keep, 1), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(lay, x, ev=None):
        xin = lay.route(x)
        if ev:
            ev[0].record()
        f, sh = lay.experts_and_shared(xin)
        if ev:
            ev[1].record()
        if kind == "refill":
            abi.razor_refill_rms_accumulate(f, lay.slot_row[:T], lay.topk_idx[:T], lay.topk_logit[:T],
                                            lay.offsets, sum_sq, count, shared_out=sh, y_out=lay.y[:T],
                                            ws=lay.ws_refill)
            abi.razor_select(sum_sq, count, wl.keep, kept=kept)
        else:
            abi.moe_combine(f, lay.slot_row[:T], lay.topk_w[:T], shared_out=sh, y=lay.y[:T])

    # one CUDA graph per unit for the timed steps, and a second set holding
    # timing events around the expert call (external event nodes, read
    # afterwards) for the expert roofline: event nodes between kernels would
    # cut the programmatic launch edges of the timed steps
    ev_pairs = [(torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n_units)]
    graphs = graphs_ev = None
    launches_per_step = None
    if not args.no_graph:
        graphs = [lay.capture(x, lambda xx, lay=lay: step(lay, xx)) for lay, x in units]
        launches_per_step = layer.graph_kernels
        graphs_ev = [lay.capture(x, lambda xx, lay=lay, ev=ev_pairs[u]: step(lay, xx, ev))
                     for u, (lay, x) in enumerate(units)]

    def run(i, with_events=False):
        u = i % n_units
        if graphs:
            (graphs_ev if with_events else graphs)[u].replay()
        else:
            step(units[u][0], units[u][1], ev_pairs[u] if with_events else None)

    for i in range(max(args.warmup, n_units)):
        run(i)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0, "device status after warm-up"

    def timed():
        dist.barrier()
        torch.cuda.synchronize()
        clocks = ClockSampler(dist.local)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            run(i)
        t_end.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        clk = clocks.stop()
        return dist.max(t_start.elapsed_time(t_end) / args.steps), clk

    ms, clk = timed()
    # a region whose clocks do not stand (on any rank) is measured once more, by every rank
    if dist.max(1.0 if clocks_rejected(clk) else 0.0) > 0:
        first = {"sm_mhz": clk["sm_mhz"], "reasons": clk["reasons"]}
        ms, clk = timed()
        clk["remeasured_after"] = first
    # expert roofline: the same rotation with events around the expert call;
    # each unit's last replay
    for i in range(max(args.steps, n_units)):
        run(i, with_events=True)
    torch.cuda.synchronize()
    ffn_ms = dist.max(statistics.mean(a.elapsed_time(b) for a, b in ev_pairs))
    # for comparison: decode steps after an L2 flush by a write of 2x L2 (the
    # flush leaves dirty lines whose write-back and the kernels' cold code
    # fall inside the step), each step timed alone, the flush excluded
    flush_ms = None
    if decode:
        l2_flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        fl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for i in range(args.steps):
            l2_flush.zero_()
            fl_ev[i][0].record(stream)
            run(i)
            fl_ev[i][1].record(stream)
        torch.cuda.synchronize()
        flush_ms = dist.max(sum(a.elapsed_time(b) for a, b in fl_ev) / args.steps)
        del l2_flush
    status = abi.moe_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    rows = T * (wl.k + extra)
    tokens = T * dist.world
    value = tokens / (ms / 1e3)
    peaks = measured_peaks()
    roofline = expert_roofline(wl, [u[0] for u in units], T, rows, ffn_ms, peaks)
    roofline["traffic"], src = measured_traffic(workload)
    if src:
        roofline["traffic_source"] = (src + ": dram__bytes_read.sum + dram__bytes_write.sum of the expert call's "
                                      "launches, bytes per call, from a one-pass ncu capture of a single-layer run of "
                                      "the same shapes (cold-cache)")

    # end-to-end through the public API: pinned host x -> y in pinned host memory, every step's upload and
    # download inside the timed region, overlapped with the neighbouring steps' forwards (HostPipeline)
    e2e = None
    if with_e2e and kind == "forward":
        xh = [x.cpu().pin_memory() for _, x in units]
        yh = [torch.empty((T, wl.H), dtype=layer.y.dtype).pin_memory() for _ in range(2)]
        pipes = {}
        for lay, _ in units:
            if id(lay) not in pipes:
                pipes[id(lay)] = HostPipeline(lay, T, use_graphs=not args.no_graph)

        def e2e_step(i):
            u = i % n_units
            pipes[id(units[u][0])].step(xh[u], yh[i & 1])

        def e2e_finish():
            for p in pipes.values():
                p.finish()

        for i in range(max(2, args.warmup, 2 * n_units)):  # every (batch, output buffer) pair once
            e2e_step(i)
        e2e_finish()
        dist.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for p in pipes.values():
            p.begin()
        for i in range(args.steps):
            e2e_step(i)
        e2e_finish()
        b.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = dist.max(a.elapsed_time(b) / args.steps)
        e2e = {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(e2e_ms, 4),
               "h2d_bytes_per_step": int(xh[0].numel() * xh[0].element_size()),
               "d2h_bytes_per_step": int(yh[0].numel() * yh[0].element_size()),
               "path": "pinned host x -> H2D copy -> layer (CUDA graph of the C-ABI calls) -> D2H copy of y, "
                       + ("one CUDA graph per step holding the upload, the forward and the download (HostPipeline, "
                          "decode-sized batch)" if T <= HostPipeline.whole_step_max_T and not args.no_graph else
                          "with HostPipeline overlapping step i+1's upload and step i-1's download with step i")}

    if launches_per_step is None:  # eager: count one pass's launches from a throw-away capture
        launches_per_step = _count_step_kernels(layer, xs[0], lambda xx: step(layer, xx))
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"bf16": "bf16", "awq_g32": f"{'bf16' if wl.act == 'bf16' else 'f16'} x int4 "
                                                                 "(AWQ g32)",
                                       "nvfp4": "fp4 e2m1 x fp4 e2m1 (NVFP4)"}[wl.fmt],
        "data": "synthetic (seeded N(0,1) tokens, N(0,1/sqrt(fan_in)) weights)",
        "config": {"workload": workload_label(workload), "tokens_per_step_per_gpu": T,
                   "parallelism": f"dp{dist.world} (replicas, no collective)",
                   "launch": "eager C-ABI calls" if args.no_graph else "one CUDA graph per step (the C-ABI calls)",
                   "l2": (f"{n_units} layers with distinct weights in rotation ({layer_bytes / 2**30:.2f} GiB each); "
                          "between two uses of a layer the others stream >= 3x the 126 MB L2 of expert weights, "
                          "so no expert weight is cached when its layer runs again; no flush" if decode else
                          f"{n_batches} rotating token batches ({n_batches * x_bytes / 2**20:.0f} MiB) and "
                          f"{layer_bytes / 2**30:.1f} GiB of expert weights per step's reach, both larger than the "
                          "126 MB L2")},
        "roofline": roofline, "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clk,
        "expert_ffn_ms": round(ffn_ms, 4),
        "ms_per_step_after_l2_write_flush": None if flush_ms is None else round(flush_ms, 4),
        "launches_per_step": launches_per_step,
    }
    roofline["timing"] = ("CUDA events around the expert call, in a second run of the same rotation right after "
                          "the timed region; mean over the units")
    if dist.rank == 0 and with_cpu:
        # the same per-call sample as the reference arm's steps (so the two
        # rates compare): one untimed call, then calls on consecutive slices
        # of one batch until about 10 s of CPU work
        n = min(args.cpu_sample_tokens or CPU_SAMPLE_TOKENS[kind], T)
        oracle_tokens_per_s(wl, w, xs[0][T - n:], n, kind)  # untimed warm-up call, as the reference arm has
        tot_t, tot_n, calls = 0.0, 0, 0
        while calls < 4 and (calls == 0 or tot_t < 10.0) and (calls + 1) * n <= T:
            _, dt = oracle_tokens_per_s(wl, w, xs[0][calls * n:], n, kind)
            tot_t += dt
            tot_n += n
            calls += 1
        line["cpu_baseline"] = {"value": round(tot_n / tot_t, 3), "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{calls} calls of {n} consecutive tokens of one batch of the same workload, "
                                          f"full layer in float64 NumPy ({tot_t:.1f} s)"}
    return line


def decode_summary(line: dict) -> dict:
    """The decode figures of one workload's line, for the default line's
    `decode` key."""
    r = line["roofline"]
    return {"tokens_per_s": line["value"], "ms_per_step": line["ms_per_step"],
            "ms_per_step_after_l2_write_flush": line["ms_per_step_after_l2_write_flush"],
            "expert_call_gbs": r["achieved"], "hbm_peak_gbs": r["peak"], "frac": r["frac"],
            "traffic": r.get("traffic"),
            "frac_of_nominal_8tbs": r["frac_of_nominal"], "work_per_launch": r["work_per_launch"],
            "expert_ffn_ms": line["expert_ffn_ms"], "launches_per_step": line["launches_per_step"],
            "clocks": line["clocks"], "l2": line["config"]["l2"]}


def run_native(args, dist: Dist) -> None:
    line = bench_workload(args, dist, args.workload, with_e2e=not args.no_e2e, with_cpu=not args.no_cpu_baseline)
    if args.workload == "bf16_prefill" and not args.no_decode:
        # the metric's decode half, measured in the same run: HBM GB/s of the
        # expert call (the distinct experts' weights) for T = 1 and T = 64
        torch.cuda.empty_cache()
        line["decode"] = {}
        for wk in DECODE_COMPANIONS:
            dl = bench_workload(args, dist, wk, with_e2e=False, with_cpu=False)
            line["decode"][wk] = decode_summary(dl)
            torch.cuda.empty_cache()
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def workload_label(workload: str) -> str:
    """The workload as both arms name it in their JSON line's config."""
    wname, T, kind = WORKLOADS[workload]
    wl = synth.WORKLOADS[wname]
    keep = PRUNED.get(workload, 0)
    label = (f"{workload}: T={T} H={wl.H} E={keep or wl.E} k={wl.k} I={wl.I} shared={wl.I_sh} fmt={wl.fmt}"
             + (" +Refill-RMS accumulate/select" if kind == "refill" else ""))
    if keep:
        label += (f" (RAZOR-pruned from {wl.E} experts: Refill-RMS over one {CALIBRATION_T}-token calibration row, "
                  f"top {keep} kept, sliced on the device)")
    return label


def run_reference(args, dist: Dist) -> None:
    """The CPU oracle as the reference arm, rank 0 only."""
    if dist.rank != 0:
        return
    wname, T, kind = WORKLOADS[args.workload]
    wl = synth.WORKLOADS[wname]
    keep = PRUNED.get(args.workload, 0)
    if keep:  # a layer of the pruned shape, seeded weights (the selection itself is not timed)
        wl = dataclasses.replace(wl, E=keep)
    dev = torch.device("cuda", dist.local) if torch.cuda.is_available() else torch.device("cpu")
    w = synth.make_weights(wl, seed=0, device=dev)
    x = synth.make_tokens(wl, T, seed=1, device=dev)
    n = min(args.cpu_sample_tokens or CPU_SAMPLE_TOKENS[kind], T)
    for _ in range(args.warmup):
        oracle_tokens_per_s(wl, w, x, n, kind)
    tot_t, tot_n = 0.0, 0
    for i in range(args.steps):
        xi = x[(i * n) % T:][:n]
        _, dt = oracle_tokens_per_s(wl, w, xi, n, kind)
        tot_t += dt
        tot_n += n
    v = tot_n / tot_t
    line = {
        "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_label(args.workload), "tokens_per_step_per_gpu": n},
        "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{n} tokens per step of the same workload, float64 NumPy"
                                   + (f" (a layer of the pruned shape, E={keep}, seeded weights)" if keep else "")},
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    dist = Dist()
    try:
        if args.impl == "reference":
            run_reference(args, dist)
        else:
            run_native(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
