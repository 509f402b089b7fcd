"""Shared helpers of the tests: tensor -> oracle input conversion and error
metrics.  No arithmetic of the method lives here."""

import numpy as np
import torch

from oracle import formats


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a BF16 / FP16 / FP32 tensor, through the oracle's
    own converters for the 16-bit formats."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return formats.bf16_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    if t.dtype == torch.float16:
        return formats.f16_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    return t.double().numpy()


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """Normwise relative error max|got - ref| / max|ref|."""
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref)) / max(np.max(np.abs(ref)), 1e-30))


def expert_fn_bf16(w: dict, I: int):
    gu = w["w_gate_up"]
    wd = w["w_down"]
    cache = {}

    def ew(e):
        if e not in cache:
            g = f64(gu[e])
            cache[e] = (g[:I], g[I:], f64(wd[e]))
        return cache[e]

    return ew


def shared_fn(w: dict):
    g = f64(w["w_sh_gate_up"])
    I = g.shape[0] // 2
    return g[:I], g[I:], f64(w["w_sh_down"])


def refill_stats_ref(ref: dict, k: int, E: int, margin: float = 1e-3):
    """Oracle Refill statistics over the decided tokens, plus the experts whose
    statistics no undecided token can touch (not in any undecided token's
    oracle top-(k+2))."""
    from oracle import moe, razor

    r = ref["route"]
    ok = r["margin"] > margin
    d = razor.refill_deltas_closed_form(ref["f"], ref["perm"]["slot_row"], r["idx"], r["p"], k)
    s = np.zeros(E)
    c = np.zeros(E, np.int64)
    razor.accumulate(s, c, d[ok], r["idx"][ok], k)
    order = moe.expert_order(r["p"])
    bad = np.unique(order[~ok, : k + 2]) if (~ok).any() else np.zeros(0, np.int64)
    good = np.setdiff1d(np.arange(E), bad)
    return s, c, good
