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


def expert_fn_bf16(w: dict, I: int, cache: bool = True):
    """e -> float64 (w_gate [I,H], w_up [I,H], w_down [H,I]) of a BF16 layer.
    cache=False converts on every call (a full E=512 bank is 16 GB of
    float64; the oracle's routed_outputs asks for each expert once)."""
    gu = w["w_gate_up"]
    wd = w["w_down"]
    store = {}

    def ew(e):
        if e in store:
            return store[e]
        g = f64(gu[e])
        out = (g[:I], g[I:], f64(wd[e]))
        if cache:
            store[e] = out
        return out

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


def tile_edge_sample(x_rows: int, perm: dict, n_total: int, seed: int, n_experts: int = 3, tile: int = 128):
    """Token indices for a sampled full-size check: every token with a row in
    the first and in the last 128-row tile of the n_experts most-loaded
    experts of the (oracle's) permutation, the first and last token, and
    random other tokens up to n_total in all; sorted, unique."""
    off = np.asarray(perm["offsets"])
    rt = np.asarray(perm["row_token"])
    counts = np.diff(off)
    top = np.argsort(-counts, kind="stable")[:n_experts]
    picks = [np.array([0, x_rows - 1])]
    for e in top:
        a, b = int(off[e]), int(off[e + 1])
        picks.append(rt[a:min(b, a + tile)])
        last = a + ((b - a - 1) // tile) * tile  # first row of the expert's last tile
        picks.append(rt[last:b])
    edge = np.unique(np.concatenate(picks))
    rest = np.setdiff1d(np.arange(x_rows), edge)
    extra = np.random.default_rng(seed).choice(rest, max(0, min(len(rest), n_total - len(edge))), replace=False)
    return np.unique(np.concatenate([edge, extra]))


def kept_set_swaps(kept_gpu, scores_ref: np.ndarray, keep: int, band: float):
    """Checks a kept set against the oracle's scores at the keep boundary.
    thr = the mean of the oracle's keep-th and (keep+1)-th scores; every
    expert scoring above thr * (1 + band) must be kept, none scoring below
    thr * (1 - band) may be; experts inside the band may swap.  Returns the
    swapped experts (the symmetric difference with the oracle's own kept
    set, each inside the band)."""
    from oracle import razor

    kept_gpu = np.asarray(kept_gpu)
    E = len(scores_ref)
    assert len(kept_gpu) == keep and len(np.unique(kept_gpu)) == keep
    assert np.all(np.diff(kept_gpu) > 0), "kept indices must be ascending"
    kept_ref = np.sort(np.lexsort((np.arange(E), -scores_ref))[:keep])
    if keep == E:
        assert np.array_equal(kept_gpu, kept_ref)
        return []
    srt = np.sort(scores_ref)[::-1]
    thr = 0.5 * (srt[keep - 1] + srt[keep])
    kg = set(kept_gpu.tolist())
    must_in = np.nonzero(scores_ref > thr * (1 + band))[0]
    must_out = np.nonzero(scores_ref < thr * (1 - band))[0]
    missing = [int(e) for e in must_in if e not in kg]
    wrong = [int(e) for e in must_out if e in kg]
    assert not missing and not wrong, (missing, wrong)
    swaps = sorted(kg.symmetric_difference(kept_ref.tolist()))
    for e in swaps:
        assert abs(scores_ref[e] - thr) <= band * thr, e
    return swaps


def _nvfp4_quantize_mats(mats):
    """Worker of nvfp4_oracle_bank (top level, so a spawned process can run
    it): BF16 bit patterns -> the oracle's quantisation of each matrix."""
    from oracle import formats, nvfp4

    return [nvfp4.quantize(formats.bf16_to_f64(m).astype(np.float32)) for m in mats]


def nvfp4_oracle_bank(w: dict, I: int, experts, workers: int = 0):
    """The oracle's own NVFP4 quantisation of a layer's BF16 expert weights
    (gate, up and down of each expert as separate tensors), for the given
    experts, computed in parallel by spawned worker processes (the oracle's
    quantiser is elementwise NumPy on one core).  Returns e -> dequantised
    float64 (w_gate, w_up, w_down), dequantising on each call."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os

    from oracle import nvfp4

    def bits(t):
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    experts = [int(e) for e in experts]
    jobs = []
    for e in experts:
        g = bits(w["w_gate_up"][e])
        jobs.append([g[:I], g[I:], bits(w["w_down"][e])])
    n = workers or max(1, min(32, (os.cpu_count() or 2) - 1))
    with cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        raw = dict(zip(experts, ex.map(_nvfp4_quantize_mats, jobs, chunksize=4)))

    def deq(e):
        return tuple(nvfp4.dequant(*q) for q in raw[int(e)])

    return deq, raw
