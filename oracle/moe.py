"""Routed-expert MoE layer of a Qwen3.8-Flash-Next-style model, float64.

Test infrastructure (see the package docstring).

Sources (page title, then the section or table entry):
* Qwen3.8-Flash-Next architecture fact sheet (archdb model page):
  "Gating function over expert logits": softmax; "Routed experts selected per
  token": 10 of 512; "Selected expert weights are renormalized to sum to 1":
  yes; "Always-on experts per MoE layer": 1, of width 640; "FFN activation":
  SwiGLU, no clamping, no bias.
* Qwen3.8-Flash-Next-RAZOR-65B-A6B-E256of512 card, opening paragraphs: expert
  weights and router rows are sliced together, so the router is an E x d_model
  row matrix.
* Qwen3.8-Flash-Next-AWQ-g32 card, "Checkpoint": the expert projections are
  gate_proj, up_proj and down_proj.

Readings where the pages are silent:
* weights are stored out x in (row j of w_gate is output feature j);
* the synthetic router bias is added to the logits before the softmax;
* ties in the expert order go to the lower expert index;
* within one expert the permuted rows are in ascending token order;
* SwiGLU is silu(gate) * up with silu(g) = g / (1 + exp(-g));
* the shared expert is added to the routed sum without a gate; the AWQ
  card lists a shared-expert gate tensor without its formula, and where one
  is given it is read as a logistic gate per token, sigmoid(x . w_gate).
"""

from __future__ import annotations

from typing import Callable, Optional, Sequence

import numpy as np

from .formats import f64_to_bf16_values


def router_logits(x: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    """l = x . Wr^T (+ b).  x [T, H], w_router [E, H], bias [E] -> [T, E]."""
    l = np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, np.float64)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (all E experts), max-subtracted."""
    m = np.max(l, axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def expert_order(p: np.ndarray) -> np.ndarray:
    """Experts of each token by descending probability, ties to the lower
    index: a full stable sort of -p."""
    return np.argsort(-p, axis=-1, kind="stable")


def route(x, w_router, bias, k: int, extra: int = 0) -> dict:
    """Router, softmax over all E, top-k, renormalised weights.

    Returns a dict with
      idx    [T, k+extra] int64   selected experts, descending p (rank k+1 last
                                  when extra == 1: the expert Refill promotes)
      w      [T, k]       float64 p_S / sum(p_S)
      p      [T, E]       float64 softmax over all experts
      logits [T, E]       float64
      margin [T]          float64 logit gap that decides the selected set
                                  (rank k vs k+1, and k+1 vs k+2 when extra)
    """
    l = router_logits(x, w_router, bias)
    p = softmax(l)
    order = expert_order(p)
    ks = k + extra
    idx = order[:, :ks]
    p_sel = np.take_along_axis(p, idx[:, :k], axis=1)
    w = p_sel / np.sum(p_sel, axis=1, keepdims=True)
    ls = np.take_along_axis(l, order, axis=1)
    E = l.shape[1]
    gaps = []
    for r in range(1, ks + (1 if ks < E else 0)):
        if r < E:
            gaps.append(ls[:, r - 1] - ls[:, r])
    # the set decision depends on every consecutive gap up to rank ks; the
    # order inside the set only changes the order of the output columns
    margin = np.min(np.stack(gaps, axis=1), axis=1) if gaps else np.full(l.shape[0], np.inf)
    if ks < E:
        boundary = ls[:, ks - 1] - ls[:, ks]
        if extra:
            boundary = np.minimum(boundary, ls[:, k - 1] - ls[:, k])
    else:
        boundary = np.full(l.shape[0], np.inf)
    return dict(idx=idx, w=w, p=p, logits=l, margin=margin, set_margin=boundary)


def permute(idx: np.ndarray, E: int) -> dict:
    """Group the (token, slot) assignments by expert.

    idx [T, ks] -> offsets [E+1] (exclusive scan of the per-expert counts),
    row_token [T*ks] (token of each permuted row), slot_row [T, ks] (permuted
    row of each assignment).  Expert blocks are in ascending expert id and the
    rows of one expert in ascending token order: a stable sort of the
    flattened expert ids.
    """
    idx = np.asarray(idx, np.int64)
    T, ks = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")  # permuted row -> flat assignment
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    row_token = order // ks
    slot_row = np.empty(T * ks, np.int64)
    slot_row[order] = np.arange(T * ks)
    return dict(offsets=offsets, row_token=row_token, slot_row=slot_row.reshape(T, ks), counts=counts)


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def swiglu_expert(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray):
    """One SwiGLU expert: h = silu(x Wg^T) * (x Wu^T), f = h Wd^T.
    x [n, H], w_gate / w_up [I, H], w_down [H, I] -> (f [n, H], h [n, I])."""
    x = np.asarray(x, np.float64)
    g = x @ np.asarray(w_gate, np.float64).T
    u = x @ np.asarray(w_up, np.float64).T
    h = silu(g) * u
    return h @ np.asarray(w_down, np.float64).T, h


def combine(f_rows: np.ndarray, slot_row: np.ndarray, w: np.ndarray, shared: Optional[np.ndarray]) -> np.ndarray:
    """y_t = sum_j w[t, j] f[slot_row[t, j]] (+ shared_t).  Only the first
    w.shape[1] slots are combined (a Refill pass carries one extra slot)."""
    T, k = w.shape
    y = np.zeros((T, f_rows.shape[1]), np.float64)
    for j in range(k):
        y += w[:, j:j + 1] * f_rows[slot_row[:, j]]
    if shared is not None:
        y += shared
    return y


def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Pre-norm RMSNorm with a (1 + w) gain (architecture fact sheet,
    normalisation entries: gain 1 + w, before the block, epsilon 1e-6): the
    MoE block's input is
    x / sqrt(mean(x^2) + eps) * (1 + w) over the hidden dimension.
    x [T, H], w [H] -> [T, H]."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * (1.0 + np.asarray(w, np.float64))


def block_input(x: np.ndarray, w: np.ndarray, eps: float = 1e-6, dtype: str = "bf16") -> np.ndarray:
    """The MoE block's input when the layer carries its pre-MoE RMSNorm: the
    normalised activation as the model's 16-bit tensor (BF16, or FP16 for
    the AWQ card's FP16 compute), rounded once from the exact value.  The
    router, the experts, the shared expert and its gate all read it.
    x [T, H], w [H] -> [T, H] float64 holding 16-bit values."""
    y = rmsnorm(x, w, eps)
    if dtype == "bf16":
        return f64_to_bf16_values(y)
    if dtype == "f16":
        return np.asarray(y, np.float64).astype(np.float16).astype(np.float64)
    raise ValueError(dtype)


def shared_gate(x: np.ndarray, w_gate: np.ndarray) -> np.ndarray:
    """Per-token shared-expert gate 1 / (1 + exp(-x . w_gate)).
    x [T, H], w_gate [H] -> [T]."""
    z = np.asarray(x, np.float64) @ np.asarray(w_gate, np.float64)
    return 1.0 / (1.0 + np.exp(-z))


ExpertFn = Callable[[int], Sequence[np.ndarray]]


def routed_outputs(x: np.ndarray, perm: dict, expert_weights: ExpertFn):
    """f for every permuted row: expert e's SwiGLU on the tokens routed to it.
    expert_weights(e) -> (w_gate [I,H], w_up [I,H], w_down [H,I]) in float64."""
    offsets, row_token = perm["offsets"], perm["row_token"]
    E = len(offsets) - 1
    f = None
    h_all = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        wg, wu, wd = expert_weights(e)
        fe, he = swiglu_expert(x[row_token[a:b]], wg, wu, wd)
        if f is None:
            f = np.zeros((len(row_token), fe.shape[1]), np.float64)
            h_all = np.zeros((len(row_token), he.shape[1]), np.float64)
        f[a:b] = fe
        h_all[a:b] = he
    return f, h_all


def moe_layer(x, w_router, bias, k: int, expert_weights: ExpertFn, shared_weights=None, extra: int = 0,
              shared_gate_w=None) -> dict:
    """The whole routed-expert layer on tokens x [T, H] (float64):
    route -> permute -> per-expert SwiGLU -> weighted combine (+ shared,
    times the per-token gate when shared_gate_w [H] is given).
    Returns route / permutation intermediates, f, h and y."""
    x = np.asarray(x, np.float64)
    E = np.asarray(w_router).shape[0]
    r = route(x, w_router, bias, k, extra)
    perm = permute(r["idx"], E)
    f, h = routed_outputs(x, perm, expert_weights)
    shared = None
    if shared_weights is not None:
        shared, _ = swiglu_expert(x, *shared_weights)
        if shared_gate_w is not None:
            shared = shared * shared_gate(x, shared_gate_w)[:, None]
    y = combine(f, perm["slot_row"], r["w"], shared)
    return dict(route=r, perm=perm, f=f, h=h, shared=shared, y=y)
