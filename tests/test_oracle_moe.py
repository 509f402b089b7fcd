"""Pins for oracle/moe.py: brute force on tiny inputs, special cases that
reduce to a dense textbook formula, torch's own softmax / silu, and
structural invariants of the permutation."""

import json
import os

import numpy as np
import torch

from oracle import moe
from bit_expert_gemm_b200 import synth


def _tiny(seed=0, T=64):
    wl = synth.WORKLOADS["tiny"]
    w = synth.make_weights(wl, seed)
    x = synth.make_tokens(wl, T, seed).double().numpy()
    wr = w["w_router"].double().numpy()
    b = w["bias"].double().numpy()
    gu = w["w_gate_up"].double().numpy()
    wd = w["w_down"].double().numpy()
    I = wl.I

    def ew(e):
        return gu[e, :I], gu[e, I:], wd[e]

    sh = (w["w_sh_gate_up"].double().numpy()[:wl.I_sh], w["w_sh_gate_up"].double().numpy()[wl.I_sh:],
          w["w_sh_down"].double().numpy())
    return wl, x, wr, b, ew, sh


def test_softmax_and_silu_vs_torch():
    rng = np.random.default_rng(0)
    l = rng.standard_normal((50, 37)) * 4
    assert np.allclose(moe.softmax(l), torch.softmax(torch.from_numpy(l), -1).numpy(), rtol=1e-13, atol=0)
    g = rng.standard_normal(1000) * 10
    assert np.allclose(moe.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(), rtol=1e-12, atol=1e-300)


def _brute_topk(row, k):
    """Iterated arg-max in pure Python, ties to the lower index."""
    left = list(range(len(row)))
    out = []
    for _ in range(k):
        best = left[0]
        for e in left[1:]:
            if row[e] > row[best]:
                best = e
        out.append(best)
        left.remove(best)
    return out


def test_route_topk_matches_brute_force_with_ties():
    wl, x, wr, b, _, _ = _tiny()
    r = moe.route(x, wr, b, k=3, extra=1)
    for t in range(x.shape[0]):
        assert list(r["idx"][t]) == _brute_topk(list(r["p"][t]), 4)
    # exact ties: equal logits must go to the lower index
    xt = np.zeros((1, 4))
    wrt = np.zeros((6, 4))
    bt = np.array([1.0, 2.0, 2.0, 0.5, 2.0, 1.0])
    rt = moe.route(xt, wrt, bt, k=4)
    assert list(rt["idx"][0]) == [1, 2, 4, 0]


def test_route_weights_sum_to_one_and_follow_probabilities():
    wl, x, wr, b, _, _ = _tiny()
    r = moe.route(x, wr, b, k=wl.k)
    assert np.allclose(r["w"].sum(1), 1.0, atol=1e-12)
    # renormalising over S equals a softmax over the selected logits only
    ls = np.take_along_axis(r["logits"], r["idx"], 1)
    assert np.allclose(r["w"], torch.softmax(torch.from_numpy(ls), -1).numpy(), rtol=1e-12)


def test_permute_structure_and_brute_force():
    idx = synth.make_routing(200, 16, 3, seed=4).numpy()
    p = moe.permute(idx, 16)
    T, ks = idx.shape
    assert np.array_equal(p["counts"], np.bincount(idx.ravel(), minlength=16))
    assert p["offsets"][0] == 0 and np.array_equal(np.diff(p["offsets"]), p["counts"])
    # bijection between (t, j) and rows, consistent with row_token
    rows = p["slot_row"].ravel()
    assert np.array_equal(np.sort(rows), np.arange(T * ks))
    for t in range(T):
        for j in range(ks):
            assert p["row_token"][p["slot_row"][t, j]] == t
    # brute force: per expert, the tokens that chose it, ascending
    pos = 0
    for e in range(16):
        toks = [t for t in range(T) if e in idx[t]]
        assert list(p["row_token"][pos:pos + len(toks)]) == toks
        pos += len(toks)


def test_layer_with_k_equal_E_is_dense_softmax_mixture():
    wl, x, wr, b, ew, _ = _tiny()
    E = wr.shape[0]
    out = moe.moe_layer(x, wr, b, E, ew)
    p = torch.softmax(torch.from_numpy(x @ wr.T + b), -1).numpy()
    dense = np.zeros_like(out["y"])
    for e in range(E):
        wg, wu, wd = ew(e)
        xt = torch.from_numpy(x)
        fe = (torch.nn.functional.silu(xt @ torch.from_numpy(wg).T) * (xt @ torch.from_numpy(wu).T)) @ torch.from_numpy(wd).T
        dense += p[:, e:e + 1] * fe.numpy()
    assert np.allclose(out["y"], dense, rtol=1e-10, atol=1e-12)


def test_single_expert_layer_is_textbook_swiglu():
    wl, x, wr, b, ew, sh = _tiny()
    out = moe.moe_layer(x, wr[:1], b[:1], 1, ew, sh)
    xt = torch.from_numpy(x)
    wg, wu, wd = (torch.from_numpy(a) for a in ew(0))
    sg, su, sd = (torch.from_numpy(a) for a in sh)
    ref = (torch.nn.functional.silu(xt @ wg.T) * (xt @ wu.T)) @ wd.T
    ref = ref + (torch.nn.functional.silu(xt @ sg.T) * (xt @ su.T)) @ sd.T
    assert np.allclose(out["y"], ref.numpy(), rtol=1e-11, atol=1e-12)


def test_only_one_nonzero_expert():
    wl, x, wr, b, ew, _ = _tiny()
    star = int(np.argmax(b))

    def ew0(e):
        wg, wu, wd = ew(e)
        return (wg, wu, wd) if e == star else (wg * 0, wu * 0, wd * 0)

    out = moe.moe_layer(x, wr, b, wl.k, ew0)
    r = out["route"]
    fstar, _ = moe.swiglu_expert(x, *ew(star))
    want = np.zeros_like(out["y"])
    for t in range(x.shape[0]):
        js = np.nonzero(r["idx"][t] == star)[0]
        if len(js):
            want[t] = r["w"][t, js[0]] * fstar[t]
    assert np.allclose(out["y"], want, rtol=1e-12, atol=1e-14)


def test_expert_structure_matches_published_parameter_counts():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "param_counts.json")))
    d, I = g["d_model"], g["expert_dim"]
    # one expert of the oracle's layer: gate [I,d], up [I,d], down [d,I]; plus its router row [d]
    shapes = [(I, d), (I, d), (d, I), (d,)]
    per_expert = sum(int(np.prod(s)) for s in shapes)
    L = g["main_moe_layers"]
    assert g["main_base"] - g["main_keep256"] == L * 256 * per_expert
    assert g["main_base"] - g["main_keep384"] == L * 128 * per_expert
    assert g["mtp_base"] - g["mtp_keep256"] == g["mtp_moe_layers"] * 256 * per_expert
    assert g["mtp_base"] - g["mtp_keep384"] == g["mtp_moe_layers"] * 128 * per_expert
    # and the assumed H = 2048 of the graded workloads would not reproduce them
    d2 = 2048
    assert g["main_base"] - g["main_keep256"] != L * 256 * (3 * d2 * I + d2)


def test_shared_gate_closed_forms_and_library():
    from scipy.special import expit

    x = np.array([[1.0, 2.0], [-3.0, 0.5], [0.0, 0.0]])
    g = np.array([0.5, -1.0])
    assert np.allclose(moe.shared_gate(x, g), expit(x @ g), rtol=1e-15)
    assert np.array_equal(moe.shared_gate(x, np.zeros(2)), np.full(3, 0.5))  # a zero gate halves the shared expert
    assert moe.shared_gate(np.array([[40.0]]), np.array([1.0]))[0] == 1.0
    assert moe.shared_gate(np.array([[-40.0]]), np.array([1.0]))[0] < 1e-17


def test_layer_with_gate_scales_only_the_shared_expert():
    wl = synth.WORKLOADS["tiny"]
    w = synth.make_weights(wl, 4)
    x = synth.make_tokens(wl, 32, 4).double().numpy()
    gu, wd = w["w_gate_up"].double().numpy(), w["w_down"].double().numpy()
    I = wl.I
    ew = lambda e: (gu[e, :I], gu[e, I:], wd[e])  # noqa: E731
    shg = w["w_sh_gate_up"].double().numpy()
    sh = (shg[:I], shg[I:], w["w_sh_down"].double().numpy())
    g = synth.make_shared_gate(wl, 4).double().numpy()
    wr, b = w["w_router"].double().numpy(), w["bias"].double().numpy()
    plain = moe.moe_layer(x, wr, b, wl.k, ew, sh)
    routed = moe.moe_layer(x, wr, b, wl.k, ew, None)
    gated = moe.moe_layer(x, wr, b, wl.k, ew, sh, shared_gate_w=g)
    s_only = plain["y"] - routed["y"]
    z = x @ g
    assert np.allclose(gated["y"], routed["y"] + s_only / (1.0 + np.exp(-z))[:, None], rtol=1e-12, atol=1e-12)
    half = moe.moe_layer(x, wr, b, wl.k, ew, sh, shared_gate_w=np.zeros_like(g))
    assert np.allclose(half["y"], routed["y"] + 0.5 * s_only, rtol=1e-12, atol=1e-12)


def test_rmsnorm_against_torch_and_closed_forms():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 64)) * 3.0
    w = rng.standard_normal(64) * 0.1
    got = moe.rmsnorm(x, w)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), weight=torch.from_numpy(1.0 + w), eps=1e-6)
    assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)
    # a constant row c: c / sqrt(c^2 + eps) * (1 + w); w = -1 silences a feature
    c = np.full((1, 8), 2.0)
    wz = np.zeros(8)
    wz[3] = -1.0
    y = moe.rmsnorm(c, wz)
    assert np.allclose(y[0, [0, 1, 2, 4]], 2.0 / np.sqrt(4.0 + 1e-6), rtol=1e-15) and y[0, 3] == 0.0
    # scale invariance away from eps
    assert np.allclose(moe.rmsnorm(1e3 * x, w), got, rtol=1e-6)  # eps / mean(x^2) is about 1e-7 here


def test_bf16_rounding_from_float64():
    """formats.f64_to_bf16_values: one round-to-nearest-even from float64 to
    BF16.  On values exact in binary32 it equals the pinned binary32
    converter; every result is a BF16 value; the error is at most half a
    BF16 ulp; exact midpoints go to the even neighbour."""
    from oracle import formats
    rng = np.random.default_rng(8)
    v32 = (rng.standard_normal(20000) * np.exp(rng.standard_normal(20000) * 3)).astype(np.float32)
    got = formats.f64_to_bf16_values(v32.astype(np.float64))
    assert np.array_equal(got, formats.bf16_to_f64(formats.f32_to_bf16(v32)))
    v = rng.standard_normal(20000) * 5.0
    r = formats.f64_to_bf16_values(v)
    assert np.array_equal(formats.bf16_to_f64(formats.f32_to_bf16(r.astype(np.float32))), r)  # representable
    ulp = np.ldexp(1.0, np.frexp(v)[1] - 8)  # spacing of BF16 values around v
    assert np.all(np.abs(r - v) <= ulp / 2)
    mids = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.0 + 2.0 ** -7])
    assert np.array_equal(formats.f64_to_bf16_values(mids), [1.0, 1.0 + 2.0 ** -6, -1.0, 3.0])


def test_block_input_is_the_rounded_norm():
    """moe.block_input: the pinned RMSNorm, rounded once to BF16 (or FP16):
    within half a 16-bit ulp of torch's rms_norm and exactly a 16-bit value."""
    from oracle import formats
    rng = np.random.default_rng(9)
    x = rng.standard_normal((9, 128)) * 2.0
    w = rng.standard_normal(128) * 0.1
    exact = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), weight=torch.from_numpy(1.0 + w),
                                         eps=1e-6).numpy()
    b = moe.block_input(x, w)
    assert np.array_equal(formats.bf16_to_f64(formats.f32_to_bf16(b.astype(np.float32))), b)
    assert np.all(np.abs(b - exact) <= np.ldexp(1.0, np.frexp(exact)[1] - 8) / 2 * (1 + 1e-12))
    assert not np.array_equal(b, exact)
    h = moe.block_input(x, w, dtype="f16")
    assert np.array_equal(h.astype(np.float16).astype(np.float64), h)
    assert np.all(np.abs(h - exact) <= np.ldexp(1.0, np.frexp(exact)[1] - 11) / 2 * (1 + 1e-12))
