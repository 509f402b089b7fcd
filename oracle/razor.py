"""RAZOR Refill-RMS expert score and selection, float64.

Test infrastructure (see the package docstring).

Source: Qwen3.8-Flash-Next-RAZOR-65B-A6B-E256of512 card (and the copy of the
same text for the 384-expert budget on the NVFP4 card), section "Selection
and calibration":
* an expert is scored by how much the layer's local output moves when that
  expert is taken out of a token's selection and the router's best
  unselected expert takes its place, aggregated as a root mean square;
* the mean runs only over the calibration tokens that selected the expert
  (neither a sum over the corpus nor a plain average);
* each layer keeps its 256 (or 384) best-scoring experts;
* the statistics add up across rows and runs (earlier ones were reused).
The opening paragraphs add that the kept experts' weights and router rows are
cut from the original checkpoint in the same order, and that the keep
manifest lists the original expert indices in the pruned layer's order.  The MTP item of the same section keeps the MTP
layer's experts by the L2 norm of their original router rows
(mtp_policy=router_norm), because the text calibration never runs that layer.

Readings where the pages are silent: "local output" is the MoE block output, so
the shared expert cancels; the change is measured with the L2 norm over the
hidden dimension and the per-expert score is sqrt(sum ||delta||^2 / count);
count[e] counts tokens whose selected set contains e (the promoted expert
earns nothing); an expert with count 0 scores 0; ties in the ranking go to the
lower index; the kept indices are returned in ascending original order.
"""

from __future__ import annotations

import numpy as np

from . import moe


def refill_deltas_literal(f_rows: np.ndarray, slot_row: np.ndarray, idx: np.ndarray, p: np.ndarray, k: int):
    """The definition, written out: for each token t and each selected expert
    e = idx[t, j] (j < k), take S' = S minus e plus the rank-(k+1) expert r,
    renormalise the router probabilities over S', and return
    delta[t, j] = sum_{S'} w' f - sum_S w f   ([T, k, H] float64).

    f_rows are the expert outputs of the permuted rows, slot_row [T, k+1]
    maps each (token, slot) to its row, p [T, E] are the full softmax
    probabilities, idx [T, k+1] the selection with r last."""
    T = idx.shape[0]
    H = f_rows.shape[1]
    out = np.zeros((T, k, H), np.float64)
    for t in range(T):
        S = list(range(k))
        pS = np.array([p[t, idx[t, j]] for j in S])
        fS = np.stack([f_rows[slot_row[t, j]] for j in S])
        y = (pS / pS.sum()) @ fS
        for j in range(k):
            slots = [s for s in S if s != j] + [k]
            pS2 = np.array([p[t, idx[t, s]] for s in slots])
            fS2 = np.stack([f_rows[slot_row[t, s]] for s in slots])
            y2 = (pS2 / pS2.sum()) @ fS2
            out[t, j] = y2 - y
    return out


def refill_deltas_closed_form(f_rows, slot_row, idx, p, k: int):
    """Same quantity through Z = sum_S p, U = sum_S p f:
    delta_e = (U - p_e f_e + p_r f_r) / (Z - p_e + p_r) - U / Z."""
    T = idx.shape[0]
    pk = np.take_along_axis(p, idx[:, : k + 1], axis=1)  # [T, k+1]
    F = f_rows[slot_row[:, : k + 1]]  # [T, k+1, H]
    Z = pk[:, :k].sum(1)
    U = np.einsum("tj,tjh->th", pk[:, :k], F[:, :k])
    y = U / Z[:, None]
    pr = pk[:, k]
    fr = F[:, k]
    out = np.empty((T, k, F.shape[2]), np.float64)
    for j in range(k):
        Zp = Z - pk[:, j] + pr
        out[:, j] = (U - pk[:, j:j + 1] * F[:, j] + pr[:, None] * fr) / Zp[:, None] - y
    return out


def refill_deltas_knockout(x, w_router, bias, k: int, expert_weights, shared_weights=None):
    """Brute force: re-evaluate the whole layer once per expert e with e
    removed from the router (its logit forced to -inf, so the router promotes
    the next expert), and take the change of y on the tokens that had
    selected e.  Returns (delta [T, k, H] ordered like the base selection,
    base layer dict).  Independent of the Refill formulas above: it only
    calls the layer itself."""
    base = moe.moe_layer(x, w_router, bias, k, expert_weights, shared_weights)
    idx = base["route"]["idx"]
    T, H = base["y"].shape
    E = np.asarray(w_router).shape[0]
    out = np.zeros((T, k, H), np.float64)
    b0 = np.zeros(E) if bias is None else np.asarray(bias, np.float64)
    for e in np.unique(idx):
        b = b0.copy()
        b[e] = -np.inf
        knocked = moe.moe_layer(x, w_router, b, k, expert_weights, shared_weights)
        rows, slots = np.nonzero(idx == e)
        out[rows, slots] = knocked["y"][rows] - base["y"][rows]
    return out, base


def accumulate(sum_sq: np.ndarray, count: np.ndarray, deltas: np.ndarray, idx: np.ndarray, k: int) -> None:
    """sum_sq[e] += ||delta||_2^2 and count[e] += 1 for every (token, selected
    expert e).  In place; additive across calls."""
    sq = np.sum(deltas * deltas, axis=2)  # [T, k]
    for j in range(k):
        np.add.at(sum_sq, idx[:, j], sq[:, j])
        np.add.at(count, idx[:, j], 1)


def scores(sum_sq: np.ndarray, count: np.ndarray) -> np.ndarray:
    """score_e = sqrt(sum_sq_e / count_e); 0 when count_e == 0."""
    s = np.zeros(len(sum_sq), np.float64)
    hit = count > 0
    s[hit] = np.sqrt(np.asarray(sum_sq, np.float64)[hit] / np.asarray(count)[hit])
    return s


def select(sum_sq: np.ndarray, count: np.ndarray, keep: int):
    """Keep the `keep` highest-scoring experts (ties: lower index first).
    Returns (kept indices ascending, full ranking, scores)."""
    s = scores(sum_sq, count)
    E = len(s)
    if not 0 <= keep <= E:
        raise ValueError("keep must be in [0, E]")
    ranking = np.lexsort((np.arange(E), -s))  # primary: -score, secondary: index
    kept = np.sort(ranking[:keep])
    return kept, ranking, s


def router_norm(w_router: np.ndarray) -> np.ndarray:
    """mtp_policy=router_norm: ||w_router[e, :]||_2 for every expert e."""
    w = np.asarray(w_router, np.float64)
    return np.sqrt(np.sum(w * w, axis=1))


def select_by_router_norm(w_router: np.ndarray, keep: int):
    """Keep the `keep` experts of largest router-row norm, ties to the lower
    index; same return values as select()."""
    w = np.asarray(w_router, np.float64)
    return select(np.sum(w * w, axis=1), np.ones(w.shape[0], np.int64), keep)


def slice_experts(a: np.ndarray, kept) -> np.ndarray:
    """The kept experts' blocks in output order: out[j] = a[kept[j]], for any
    tensor whose leading axis is the expert index (router rows, bias, expert
    weights)."""
    a = np.asarray(a)
    out = np.empty((len(kept),) + a.shape[1:], a.dtype)
    for j, e in enumerate(kept):
        out[j] = a[int(e)]
    return out
