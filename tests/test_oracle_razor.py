"""Pins for oracle/razor.py: the Refill definition against a brute-force
knock-out re-evaluation of the whole layer, the closed form against the
definition, degenerate cases, additivity, and selection against Python's
sorted()."""

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
