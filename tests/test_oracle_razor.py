"""Pins for oracle/razor.py: the Refill definition against a brute-force
knock-out re-evaluation of the whole layer, the closed form against the
definition, degenerate cases, additivity, selection against Python's
sorted(), the router-norm policy against hand values and numpy.linalg.norm,
and slicing against the unsliced layer with the removed experts masked."""

import numpy as np

from oracle import moe, razor
from bit_expert_gemm_b200 import synth


def _tiny_layer(seed=0, T=64):
    wl = synth.WORKLOADS["tiny"]
    w = synth.make_weights(wl, seed)
    x = synth.make_tokens(wl, T, seed).double().numpy()
    gu = w["w_gate_up"].double().numpy()
    wd = w["w_down"].double().numpy()
    I = wl.I
    sh = (w["w_sh_gate_up"].double().numpy()[:I], w["w_sh_gate_up"].double().numpy()[I:], w["w_sh_down"].double().numpy())
    return wl, x, w["w_router"].double().numpy(), w["bias"].double().numpy(), (lambda e: (gu[e, :I], gu[e, I:], wd[e])), sh


def test_refill_definition_equals_knockout_reevaluation():
    wl, x, wr, b, ew, sh = _tiny_layer()
    k = wl.k
    ko, base = razor.refill_deltas_knockout(x, wr, b, k, ew, sh)
    full = moe.moe_layer(x, wr, b, k, ew, sh, extra=1)
    lit = razor.refill_deltas_literal(full["f"], full["perm"]["slot_row"], full["route"]["idx"], full["route"]["p"], k)
    assert np.array_equal(full["route"]["idx"][:, :k], base["route"]["idx"])
    assert np.allclose(lit, ko, rtol=1e-9, atol=1e-12)
    assert np.abs(ko).max() > 1e-3  # the check is not vacuous


def test_refill_closed_form_equals_definition():
    wl, x, wr, b, ew, sh = _tiny_layer(seed=1)
    full = moe.moe_layer(x, wr, b, 2, ew, None, extra=1)
    args = (full["f"], full["perm"]["slot_row"], full["route"]["idx"], full["route"]["p"], 2)
    assert np.allclose(razor.refill_deltas_closed_form(*args), razor.refill_deltas_literal(*args), rtol=1e-10, atol=1e-13)


def test_refill_zero_when_promoted_expert_equals_removed():
    wl, x, wr, b, ew, _ = _tiny_layer()
    same = ew(0)
    full = moe.moe_layer(x, wr, b, wl.k, lambda e: same, None, extra=1)
    d = razor.refill_deltas_literal(full["f"], full["perm"]["slot_row"], full["route"]["idx"], full["route"]["p"], wl.k)
    assert np.abs(d).max() <= 1e-12 * np.abs(full["f"]).max()


def test_accumulation_is_additive_across_chunks():
    wl, x, wr, b, ew, _ = _tiny_layer()
    full = moe.moe_layer(x, wr, b, wl.k, ew, None, extra=1)
    r, perm = full["route"], full["perm"]
    d = razor.refill_deltas_closed_form(full["f"], perm["slot_row"], r["idx"], r["p"], wl.k)
    E = wr.shape[0]
    s1, c1 = np.zeros(E), np.zeros(E, np.int64)
    razor.accumulate(s1, c1, d, r["idx"], wl.k)
    s2, c2 = np.zeros(E), np.zeros(E, np.int64)
    for a in range(0, x.shape[0], 13):
        razor.accumulate(s2, c2, d[a:a + 13], r["idx"][a:a + 13], wl.k)
    assert np.array_equal(c1, c2) and np.allclose(s1, s2, rtol=1e-13)
    assert c1.sum() == x.shape[0] * wl.k  # the promoted expert earns no count


def test_select_hand_example_and_brute_force():
    kept, ranking, s = razor.select(np.array([4.0, 9.0, 0.0, 9.0]), np.array([1, 1, 0, 1]), 2)
    assert list(s) == [2.0, 3.0, 0.0, 3.0]
    assert list(ranking) == [1, 3, 0, 2] and list(kept) == [1, 3]
    for seed in range(5):
        ss, cc = synth.make_refill_stats(512, seed)
        ss, cc = ss.numpy(), cc.numpy()
        for keep in (0, 1, 256, 384, 512):
            kept, ranking, sc = razor.select(ss, cc, keep)
            sc_py = [(float(np.sqrt(ss[e] / cc[e])) if cc[e] else 0.0) for e in range(512)]
            brute = sorted(range(512), key=lambda e: (-sc_py[e], e))
            assert list(ranking) == brute
            assert list(kept) == sorted(brute[:keep])


def test_router_norm_hand_example_and_library():
    w = np.zeros((4, 8))
    w[0, :2] = (3.0, 4.0)   # norm 5
    w[2, 5] = -1.0          # norm 1
    w[3, :] = 0.5           # norm sqrt(8 * 0.25) = sqrt(2)
    assert np.allclose(razor.router_norm(w), [5.0, 0.0, 1.0, np.sqrt(2.0)], rtol=1e-15)
    wr = synth.make_weights(synth.WORKLOADS["tiny"], 3)["w_router"].double().numpy()
    assert np.allclose(razor.router_norm(wr), np.linalg.norm(wr, axis=1), rtol=1e-13)
    kept, ranking, s = razor.select_by_router_norm(w, 2)
    assert list(ranking) == [0, 3, 2, 1] and list(kept) == [0, 3]
    # ties go to the lower index, kept indices come out ascending
    w2 = np.array([[1.0, 0.0], [0.0, 2.0], [0.0, -1.0], [2.0, 0.0]])
    kept, ranking, _ = razor.select_by_router_norm(w2, 3)
    assert list(ranking) == [1, 3, 0, 2] and list(kept) == [0, 1, 3]
    n = np.linalg.norm(wr, axis=1)
    for keep in (1, 5, 8, 16):
        kept, _, _ = razor.select_by_router_norm(wr, keep)
        assert list(kept) == sorted(sorted(range(len(n)), key=lambda e: (-n[e], e))[:keep])


def test_sliced_layer_equals_layer_with_removed_experts_masked():
    """Slicing router rows, bias and expert weights with the same kept list
    gives the layer whose removed experts can never be selected: the pruned
    layer equals the original with the removed experts' logits at -inf (the
    renormalised weights over the selected set do not depend on the softmax
    denominator).  A slice of the router rows in another order than the
    expert weights fails it."""
    wl, x, wr, b, ew, sh = _tiny_layer(seed=2)
    E = wr.shape[0]
    kept = np.array([0, 2, 3, 5, 8, 9, 12, 15])
    wr_s, b_s = razor.slice_experts(wr, kept), razor.slice_experts(b, kept)
    gu_e = np.stack([np.concatenate(ew(e)[:2]) for e in range(E)])
    wd_e = np.stack([ew(e)[2] for e in range(E)])
    gu_s, wd_s = razor.slice_experts(gu_e, kept), razor.slice_experts(wd_e, kept)
    I = wl.I
    sliced = moe.moe_layer(x, wr_s, b_s, wl.k, lambda j: (gu_s[j, :I], gu_s[j, I:], wd_s[j]), sh)
    masked_b = np.full(E, -np.inf)
    masked_b[kept] = b[kept]
    masked = moe.moe_layer(x, wr, masked_b, wl.k, ew, sh)
    assert np.array_equal(kept[sliced["route"]["idx"]], masked["route"]["idx"])
    assert np.allclose(sliced["y"], masked["y"], rtol=1e-12, atol=1e-12)
    # the sliced router rows are the kept rows, in output order
    for j, e in enumerate(kept):
        assert np.array_equal(wr_s[j], wr[e]) and b_s[j] == b[e]
    # a mismatched order between router rows and expert weights is caught
    bad = moe.moe_layer(x, wr_s[::-1].copy(), b_s[::-1].copy(), wl.k,
                        lambda j: (gu_s[j, :I], gu_s[j, I:], wd_s[j]), sh)
    assert not np.allclose(bad["y"], masked["y"], rtol=1e-6, atol=1e-6)
