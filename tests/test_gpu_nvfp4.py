"""NVFP4 W4A4 experts on the GPU against the oracle: the quantiser (codes,
block scales, global scales) bit for bit, the grouped block-scaled SwiGLU
and whole layers within the 5e-2 normwise bound of the 4-bit paths (the
oracle computes in float64 with its own quantisation of the same BF16
weights and activations)."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from bit_expert_gemm_b200.layer import prepare_nvfp4_weights
from oracle import moe, nvfp4
from tests.helpers import f64, nvfp4_oracle_bank, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_4BIT = 5e-2


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("B,R,K,static", [(3, 7, 64, False), (1, 300, 2048, False), (2, 33, 640, False),
                                          (2, 50, 256, True), (1, 1, 16, False)])
def test_nvfp4_quantize_bit_exact(B, R, K, static):
    g = torch.Generator(device="cpu").manual_seed(B * 1000 + K)
    v = (torch.randn((B, R, K), generator=g) * torch.exp(torch.randn((B, R, 1), generator=g))).to(torch.bfloat16)
    v[0, 0, :16] = 0  # an all-zero block
    if K >= 32:
        v[0, 0, 16:32] = -1e-6  # tiny negatives: codes round to (negative) zero
    gs_in = torch.tensor([0.01 * (b + 1) for b in range(B)], dtype=torch.float32) if static else None
    codes, sf, gs = abi.moe_nvfp4_quantize(v.to(DEV), global_scale_in=None if gs_in is None else gs_in.to(DEV))
    torch.cuda.synchronize()
    for b in range(B):
        vb = f64(v[b]).astype(np.float32)
        c, sb, s_g = nvfp4.quantize(vb, None if gs_in is None else np.float32(gs_in[b]))
        assert _np(gs)[b] == s_g
        assert np.array_equal(_np(sf[b]), sb)
        assert np.array_equal(_np(codes[b]), nvfp4.pack(c))


def _case(T, H, I, E, k, seed):
    wl = dataclasses.replace(synth.WORKLOADS["nvfp4"], H=H, I=I, E=E, k=k)
    w = synth.make_weights(wl, seed=seed, device=DEV)
    x = synth.make_tokens(wl, T, seed=seed, device=DEV)
    return wl, prepare_nvfp4_weights(w), x


def _oracle_deq(w):
    """The oracle's per-(expert, projection) dequantised weights, computed
    only for the experts a batch touches (the full bank is gigabytes of
    float64)."""
    I = w["w_gate_up"].shape[1] // 2
    cache = {}

    def deq(e):
        if e not in cache:
            gu, wd = f64(w["w_gate_up"][e]), f64(w["w_down"][e])
            cache[e] = tuple(nvfp4.dequant(*nvfp4.quantize(m.astype(np.float32))) for m in (gu[:I], gu[I:], wd))
        return cache[e]

    def raw(e, name):
        gu = f64(w["w_gate_up"][e])
        m = {"gate": gu[:I], "up": gu[I:], "down": f64(w["w_down"][e])}[name]
        return nvfp4.quantize(m.astype(np.float32))

    return deq, raw


@pytest.mark.parametrize("T,H,I,E,k", [(37, 256, 128, 8, 2), (300, 512, 640, 16, 4), (1000, 2048, 640, 64, 10),
                                       (5, 2048, 640, 256, 10)])
def test_grouped_swiglu_nvfp4(T, H, I, E, k):
    wl, w, x = _case(T, H, I, E, k, seed=T + E)
    idx = synth.make_routing(T, E, k, seed=T)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    gs_out = torch.empty(2, dtype=torch.float32, device=DEV)
    f = abi.moe_grouped_swiglu_nvfp4(x, rt, off, T * k, w["w_gu"], w["sf_gu"], w["gs_gu"], w["w_d"], w["sf_d"],
                                     w["gs_d"], act_gs_out=gs_out, out_fp32=True)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    deq, raw = _oracle_deq(w)
    # the library's weight quantisation equals the oracle's, bit for bit
    c, sb, s_g = raw(0, "up")
    assert np.array_equal(_np(w["w_gu"][0, I:]), nvfp4.pack(c)) and np.array_equal(_np(w["sf_gu"][0, I:]), sb)
    assert _np(w["gs_gu"])[0, 1] == s_g
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    ref, _, (s_x, s_h) = nvfp4.routed_outputs_w4a4(f64(x), perm, deq)
    assert _np(gs_out)[0] == s_x  # x's global scale is exact (amax is order-free)
    assert abs(_np(gs_out)[1] / s_h - 1) < 1e-2
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err <= TOL_4BIT, err
    # weight scales rearranged once up front give the same result, bit for bit
    fp = abi.moe_grouped_swiglu_nvfp4_prepacked(x, rt, off, T * k, w["w_gu"], w["sfp_gu"], w["gs_gu"], w["w_d"],
                                                w["sfp_d"], w["gs_d"], out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(fp, f)


def _layer_ref(wl, w, x, deq, act_gs=None):
    xs = f64(x)
    r = moe.route(xs, f64(w["w_router"]), f64(w["bias"]), wl.k)
    perm = moe.permute(r["idx"], wl.E)
    f, _, _ = nvfp4.routed_outputs_w4a4(xs, perm, deq, act_gs)
    sh, _ = moe.swiglu_expert(xs, *shared_fn(w))
    return r, moe.combine(f, perm["slot_row"], r["w"], sh)


def test_nvfp4_layer_small_dynamic_scales():
    wl, w, x = _case(256, 512, 128, 16, 4, seed=3)
    layer = MoELayer(w, wl.k, "nvfp4", T_max=256)
    y = layer.forward(x)
    deq, _ = _oracle_deq(w)
    r, yref = _layer_ref(wl, w, x, deq)
    ok = r["margin"] > 1e-3
    err = rel_err(f64(y)[ok], yref[ok])
    assert err <= TOL_4BIT, err


def test_nvfp4_layer_prefill_sampled_static_scales():
    """Full prefill batch of the pruned NVFP4 layer (E=256, T=16384).  With
    static activation scales every token is independent, so 16 sampled tokens
    are recomputed one by one by the oracle."""
    wl = synth.WORKLOADS["nvfp4"]
    w = prepare_nvfp4_weights(synth.make_weights(wl, seed=0, device=DEV))
    x = synth.make_tokens(wl, wl.T_prefill, seed=0, device=DEV)
    s_x = np.float32(np.float32(np.abs(f64(x)).max()) / np.float32(2688.0))
    s_h = np.float32(0.006)
    w["act_gs"] = torch.tensor([s_x, s_h], dtype=torch.float32, device=DEV)
    layer = MoELayer(w, wl.k, "nvfp4", T_max=wl.T_prefill)
    y = layer.forward(x)
    torch.cuda.synchronize()
    sample = np.concatenate([np.random.default_rng(2).choice(wl.T_prefill, 14, replace=False), [0, wl.T_prefill - 1]])
    xs = x[torch.as_tensor(sample, device=DEV)]
    r0 = moe.route(f64(xs), f64(w["w_router"]), f64(w["bias"]), wl.k)
    used = np.unique(r0["idx"])
    deq_cache = {}

    def deq(e):
        if e not in deq_cache:
            gu, wd = f64(w["w_gate_up"][e]), f64(w["w_down"][e])
            I = wl.I
            deq_cache[e] = tuple(nvfp4.fake_quant(m.astype(np.float32)) for m in (gu[:I], gu[I:], wd))
        return deq_cache[e]

    assert len(used) > 0
    r, yref = _layer_ref(wl, w, xs, deq, act_gs=(s_x, s_h))
    ok = r["margin"] > 1e-3
    err = rel_err(f64(y)[sample][ok], yref[ok])
    assert err <= TOL_4BIT, err
    assert abi.moe_device_status() == 0


@pytest.mark.slow
def test_nvfp4_layer_prefill_full_dynamic_scales():
    """The NVFP4 workload at full size with the layer's own dynamic
    activation scales, exactly as the bench runs it (E=256, T=16384, top-10).
    The float64 oracle quantises the weights itself, takes s_x from all of x
    and s_h from the whole BF16-rounded intermediate of all 163,840 permuted
    rows, and computes every token's output; x's global scale must match bit
    for bit, h's within 1e-2 (its amax is one FP32 sum per element, summed in
    another order), and every decided token's output within 5e-2."""
    wl = synth.WORKLOADS["nvfp4"]
    T = wl.T_prefill
    w = prepare_nvfp4_weights(synth.make_weights(wl, seed=0, device=DEV))
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    layer = MoELayer(w, wl.k, "nvfp4", T_max=T)
    y = layer.forward(x).clone()
    # the same expert call on the layer's own routing, now also reporting the
    # activation scales it derived (the layer's call does not ask for them)
    rows = T * wl.k
    gs_out = torch.empty(2, dtype=torch.float32, device=DEV)
    f2 = abi.moe_grouped_swiglu_nvfp4_prepacked(x, layer.row_token[:rows], layer.offsets, rows, w["w_gu"],
                                                w["sfp_gu"], w["gs_gu"], w["w_d"], w["sfp_d"], w["gs_d"],
                                                act_gs_out=gs_out, out_fp32=layer.f.dtype == torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(f2, layer.f[:rows])
    assert abi.moe_device_status() == 0
    xs = f64(x)
    r = moe.route(xs, f64(w["w_router"]), f64(w["bias"]), wl.k)
    perm = moe.permute(r["idx"], wl.E)
    deq, _ = nvfp4_oracle_bank(w, wl.I, np.nonzero(perm["counts"])[0])
    f, _, (s_x, s_h) = nvfp4.routed_outputs_w4a4(xs, perm, deq)
    g = _np(gs_out)
    assert g[0] == s_x
    assert abs(g[1] / s_h - 1) < 1e-2, (g[1], s_h)
    sh, _ = moe.swiglu_expert(xs, *shared_fn(w))
    yref = moe.combine(f, perm["slot_row"], r["w"], sh)
    ok = r["margin"] > 1e-3
    assert ok.sum() >= 1024
    err = rel_err(f64(y)[ok], yref[ok])
    assert err <= TOL_4BIT, err
