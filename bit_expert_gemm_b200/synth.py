"""Seeded synthetic inputs for the MoE-layer workloads.

This module only draws random numbers: it holds none of the method's
arithmetic (no routing, no quantisation, no packing arithmetic).  It is the
one piece shared by the CUDA path's tests and bench and by the CPU oracle's
callers: both receive the same tensors.

Distributions follow the workload descriptions, reading N(0, s) as a normal
with standard deviation s: activations N(0, 1); weights N(0, 1/sqrt(fan_in));
router bias N(0, 1) (tiny layer) or N(0, 1.5) (skewed, Zipf-like load).  AWQ
codes and zero points are uniform on 0..15 -- drawn directly as random 32-bit
words, since eight uniform nibbles are one uniform word -- and AWQ scales are
|N(0, 0.02)| rounded to FP16.  NVFP4 weights are drawn as BF16 N(0,
1/sqrt(fan_in)) and quantised by whichever side consumes them.

Draw order (one torch.Generator per call, seeded with `seed`): router
weight, router bias, gate/up weights expert by expert, down weights expert
by expert, shared gate/up, shared down.  Token batches use their own
generator seeded from (seed, T, batch) so decode and prefill batches differ.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    E: int
    k: int
    I: int
    I_sh: int
    bias_std: float
    fmt: str  # "bf16" | "awq_g32" | "nvfp4"
    act: str  # "bf16" | "f16"
    T_prefill: int
    T_decode: Tuple[int, ...] = ()
    keep: int = 0  # Refill: experts kept per layer


WORKLOADS: Dict[str, Workload] = {
    # tiny layer: FP32/FP64 oracle vs BF16 GPU
    "tiny": Workload("tiny", H=256, E=16, k=2, I=64, I_sh=64, bias_std=1.0, fmt="bf16", act="bf16", T_prefill=64),
    # BF16 routed layer at Flash-Next shape (H assumed 2048)
    "bf16": Workload("bf16", H=2048, E=512, k=10, I=640, I_sh=640, bias_std=1.5, fmt="bf16", act="bf16",
                     T_prefill=8192, T_decode=(1, 8, 64)),
    # AWQ W4A16 g32 experts, FP16 activations, FP16 router and shared expert
    "awq_g32": Workload("awq_g32", H=2048, E=512, k=10, I=640, I_sh=640, bias_std=1.5, fmt="awq_g32", act="f16",
                        T_prefill=8192, T_decode=(1, 8, 32)),
    # the same AWQ experts in the BF16 mode: BF16 activations, router and shared
    # expert; the FP16 scales are rounded to BF16 by the kernels
    "awq_g32_bf16": Workload("awq_g32_bf16", H=2048, E=512, k=10, I=640, I_sh=640, bias_std=1.5, fmt="awq_g32",
                             act="bf16", T_prefill=8192, T_decode=(1, 8, 32)),
    # NVFP4 W4A4 experts of a 50%-pruned layer; BF16 router and shared expert
    "nvfp4": Workload("nvfp4", H=2048, E=256, k=10, I=640, I_sh=640, bias_std=1.5, fmt="nvfp4", act="bf16",
                      T_prefill=16384),
    # RAZOR Refill-RMS scoring pass: one packed row of 32768 tokens
    "refill": Workload("refill", H=2048, E=512, k=10, I=640, I_sh=640, bias_std=1.5, fmt="bf16", act="bf16",
                       T_prefill=32768, keep=256),
    # small case of the prefill kernels, sized for full profiler captures
    "profile_e64": Workload("profile_e64", H=2048, E=64, k=10, I=640, I_sh=640, bias_std=1.5, fmt="bf16", act="bf16",
                            T_prefill=2048),
    # extra, non-graded: the residual width the model's fact sheet states
    "bf16_h2560": Workload("bf16_h2560", H=2560, E=512, k=10, I=640, I_sh=640, bias_std=1.5, fmt="bf16",
                           act="bf16", T_prefill=8192),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std, dtype, device, chunk_rows: Optional[int] = None):
    """N(0, std) rounded to dtype; drawn in chunks along dim 0 to bound the
    float32 temporary."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n0 = shape[0]
    step = chunk_rows or n0
    for a in range(0, n0, step):
        b = min(n0, a + step)
        t = torch.randn((b - a, *shape[1:]), generator=g, device=device, dtype=torch.float32)
        out[a:b] = (t * std).to(dtype)
    return out


def _words(g, shape, device):
    """Uniform random 32-bit words (eight uniform nibbles each)."""
    return torch.randint(-(2 ** 31), 2 ** 31, shape, generator=g, device=device, dtype=torch.int64).to(torch.int32)


def _dt(name: str):
    return {"bf16": torch.bfloat16, "f16": torch.float16}[name]


def make_weights(wl: Workload, seed: int = 0, device="cpu", E: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All parameters of one MoE layer of workload wl.

    Keys: w_router [E,H], bias [E] f32, w_sh_gate_up [2*I_sh, H],
    w_sh_down [H, I_sh] (router / shared expert in the activation dtype), and
    per format:
      bf16 / nvfp4: w_gate_up [E, 2I, H] (rows 0..I-1 gate, I..2I-1 up) and
                    w_down [E, H, I], BF16, out x in;
      awq_g32:      qw_gu [E, H, 2I/8] i32, qz_gu [E, H/32, 2I/8] i32,
                    sc_gu [E, H/32, 2I] f16, qw_d [E, I, H/8] i32,
                    qz_d [E, I/32, H/8] i32, sc_d [E, I/32, H] f16.
    """
    E = wl.E if E is None else E
    H, I, Ish = wl.H, wl.I, wl.I_sh
    adt = _dt(wl.act)
    g = _gen(seed, device)
    w: Dict[str, torch.Tensor] = {}
    w["w_router"] = _normal(g, (E, H), H ** -0.5, adt, device)
    w["bias"] = torch.randn((E,), generator=g, device=device, dtype=torch.float32) * wl.bias_std
    chunk = max(1, (1 << 27) // (2 * I * H))
    if wl.fmt in ("bf16", "nvfp4"):
        w["w_gate_up"] = _normal(g, (E, 2 * I, H), H ** -0.5, torch.bfloat16, device, chunk)
        w["w_down"] = _normal(g, (E, H, I), I ** -0.5, torch.bfloat16, device, chunk)
    elif wl.fmt == "awq_g32":
        w["qw_gu"] = _words(g, (E, H, 2 * I // 8), device)
        w["qz_gu"] = _words(g, (E, H // 32, 2 * I // 8), device)
        w["sc_gu"] = (torch.randn((E, H // 32, 2 * I), generator=g, device=device) * 0.02).abs().to(torch.float16)
        w["qw_d"] = _words(g, (E, I, H // 8), device)
        w["qz_d"] = _words(g, (E, I // 32, H // 8), device)
        w["sc_d"] = (torch.randn((E, I // 32, H), generator=g, device=device) * 0.02).abs().to(torch.float16)
    else:
        raise ValueError(wl.fmt)
    w["w_sh_gate_up"] = _normal(g, (2 * Ish, H), H ** -0.5, adt, device)
    w["w_sh_down"] = _normal(g, (H, Ish), Ish ** -0.5, adt, device)
    return w


def make_shared_gate(wl: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """Optional shared-expert gate vector [H] ~ N(0, 1/sqrt(H)) in the
    activation dtype, from its own generator (the layer's other draws are
    unchanged by it)."""
    g = _gen(7_777_777 + seed, device)
    return _normal(g, (wl.H,), wl.H ** -0.5, _dt(wl.act), device)


def make_norm_weight(wl: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """Optional pre-MoE RMSNorm gain offset w [H] ~ N(0, 0.1) (the gain is
    1 + w) in the activation dtype, from its own generator."""
    g = _gen(8_888_887 + seed, device)
    return _normal(g, (wl.H,), 0.1, _dt(wl.act), device)


def make_tokens(wl: Workload, T: int, seed: int = 0, batch: int = 0, device="cpu") -> torch.Tensor:
    """x [T, H] ~ N(0, 1) in the workload's activation dtype."""
    g = _gen(1_000_003 * (seed + 1) + 7919 * T + 104_729 * batch, device)
    return _normal(g, (T, wl.H), 1.0, _dt(wl.act), device)


def make_routing(T: int, E: int, k_slots: int, seed: int = 0, skew: float = 1.5, device="cpu") -> torch.Tensor:
    """A synthetic selection for testing the permutation and the grouped GEMMs
    in isolation: k_slots distinct experts per token, drawn without
    replacement with Zipf-like expert popularity (weights exp(skew * z),
    z ~ N(0,1) per expert).  int32 [T, k_slots]."""
    g = _gen(31 * seed + 5, "cpu")
    pop = torch.exp(torch.randn((E,), generator=g) * skew)
    probs = pop.expand(T, E).contiguous()
    idx = torch.multinomial(probs, k_slots, replacement=False, generator=g)
    return idx.to(torch.int32).to(device)


def make_weights_topk(T: int, k: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Positive combine weights [T, k] float32 (uniform(0.05, 1)); the test
    that uses them passes them to both sides unchanged."""
    g = _gen(97 * seed + 3, "cpu")
    return (torch.rand((T, k), generator=g) * 0.95 + 0.05).to(device)


def make_refill_stats(E: int, seed: int = 0, zero_frac: float = 0.2, device="cpu"):
    """Synthetic accumulated Refill statistics for testing selection alone:
    sum_sq [E] f64 >= 0 and count [E] i64 with about zero_frac zeros, plus a
    few exact duplicates so that ties occur."""
    g = _gen(131 * seed + 11, "cpu")
    count = torch.randint(1, 5000, (E,), generator=g, dtype=torch.int64)
    count[torch.rand((E,), generator=g) < zero_frac] = 0
    sum_sq = torch.rand((E,), generator=g, dtype=torch.float64) * count.to(torch.float64) * 4.0
    sum_sq[count == 0] = 0.0
    if E >= 8:  # exact ties: copy a few (sum_sq, count) pairs onto other experts
        src = torch.randint(0, E, (E // 8,), generator=g)
        dst = torch.randint(0, E, (E // 8,), generator=g)
        sum_sq[dst] = sum_sq[src]
        count[dst] = count[src]
    return sum_sq.to(device), count.to(device)
