"""NVFP4 W4A4 decode batches (T <= 16) on the GPU: the CUDA-core GEMVs with
exact integer group products against the oracle's W4A4 expert math, within
the 5e-2 normwise bound of the 4-bit paths; the activation global scales
against the oracle's; static scales; a whole decode layer."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from bit_expert_gemm_b200.layer import prepare_nvfp4_weights
from oracle import moe, nvfp4
from tests.helpers import f64, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_4BIT = 5e-2


def _np(t):
    return t.detach().cpu().numpy()


def _lazy_deq(w, I):
    """Dequantised weights of the experts the batch touches only: gate, up
    and down each quantised as one tensor with its own global scale (the
    oracle's per-(expert, projection) reading)."""
    cache = {}

    def deq(e):
        if e not in cache:
            gu, wd = f64(w["w_gate_up"][e]), f64(w["w_down"][e])
            cache[e] = tuple(nvfp4.fake_quant(m.astype(np.float32)) for m in (gu[:I], gu[I:], wd))
        return cache[e]

    return deq


@pytest.mark.parametrize("T,H,I,E,k,out_fp32,static", [
    (1, 2048, 640, 256, 10, False, False),
    (1, 2048, 640, 256, 10, True, True),
    (2, 512, 128, 16, 4, True, False),
    (3, 256, 256, 8, 2, False, False),
    (8, 2048, 640, 256, 10, True, False),
    (16, 1024, 384, 64, 6, True, False),
    (16, 512, 128, 4, 3, False, True),   # many tokens per expert (n_e up to 16)
    (5, 2560, 640, 32, 10, True, False),  # the fact sheet's residual width
])
def test_nvfp4_decode_experts(T, H, I, E, k, out_fp32, static):
    wl = dataclasses.replace(synth.WORKLOADS["nvfp4"], H=H, I=I, E=E, k=k)
    w = prepare_nvfp4_weights(synth.make_weights(wl, seed=T + H + E, device=DEV))
    x = synth.make_tokens(wl, T, seed=T + 7, device=DEV)
    idx = synth.make_routing(T, E, k, seed=T + 8)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    deq = _lazy_deq(w, I)
    act_gs = None
    gs_in = None
    if static:
        s_x = np.float32(np.float32(np.abs(f64(x)).max()) / np.float32(2688.0))
        act_gs = (s_x, np.float32(0.004))
        gs_in = torch.tensor(act_gs, dtype=torch.float32, device=DEV)
    gs_out = torch.empty(2, dtype=torch.float32, device=DEV)
    f = abi.moe_grouped_swiglu_nvfp4_prepacked(x, rt, off, T * k, w["w_gu"], w["sfp_gu"], w["gs_gu"], w["w_d"],
                                               w["sfp_d"], w["gs_d"], act_gs_in=gs_in, act_gs_out=gs_out,
                                               out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    ref, _, (s_x_ref, s_h_ref) = nvfp4.routed_outputs_w4a4(f64(x), perm, deq, act_gs)
    assert _np(gs_out)[0] == np.float32(s_x_ref)
    if static:
        assert _np(gs_out)[1] == np.float32(act_gs[1])
    else:
        assert abs(_np(gs_out)[1] / s_h_ref - 1) < 1e-2
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err <= TOL_4BIT, err
    # the raw (row-major) weight scales give the same result, bit for bit
    f2 = abi.moe_grouped_swiglu_nvfp4(x, rt, off, T * k, w["w_gu"], w["sf_gu"], w["gs_gu"], w["w_d"], w["sf_d"],
                                      w["gs_d"], act_gs_in=gs_in, out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert torch.equal(f2, f)


@pytest.mark.parametrize("T", [1, 8])
def test_nvfp4_decode_layer(T):
    """The pruned NVFP4 layer (E=256, H=2048) at decode sizes, routed + shared
    experts + combine, against the oracle layer."""
    wl = synth.WORKLOADS["nvfp4"]
    w = prepare_nvfp4_weights(synth.make_weights(wl, seed=1, device=DEV))
    x = synth.make_tokens(wl, T, seed=9, device=DEV)
    layer = MoELayer(w, wl.k, "nvfp4", T_max=T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    xs = f64(x)
    r = moe.route(xs, f64(w["w_router"]), f64(w["bias"]), wl.k)
    used = np.unique(r["idx"])
    deq = _lazy_deq(w, wl.I)
    assert len(used) >= wl.k
    perm = moe.permute(r["idx"], wl.E)
    f, _, _ = nvfp4.routed_outputs_w4a4(xs, perm, deq)
    sh, _ = moe.swiglu_expert(xs, *shared_fn(w))
    yref = moe.combine(f, perm["slot_row"], r["w"], sh)
    ok = r["margin"] > 1e-3
    assert ok.any()
    assert rel_err(f64(y)[ok], yref[ok]) <= TOL_4BIT
    assert abi.moe_device_status() == 0
