"""The BF16 mode of the AWQ W4A16 g32 experts (the AWQ card's stock-runtime
paragraph: FP16 scales rounded to BF16 on load, BF16 arithmetic) on the GPU
against the oracle's BF16-mode dequantisation: weights bit for bit, expert
calls and whole layers within the 2e-2 normwise bound of the BF16 paths."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from oracle import awq, moe
from tests.helpers import f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


def _np(t):
    return t.detach().cpu().numpy()


def _wl(**kw):
    return dataclasses.replace(synth.WORKLOADS["awq_g32_bf16"], **kw)


@pytest.mark.parametrize("E,K,N", [(3, 64, 64), (2, 2048, 1280), (2, 640, 2048), (1, 96, 24)])
def test_awq_dequant_bf16_bit_exact(E, K, N):
    w = synth.make_weights(_wl(H=K, I=N // 2, E=E), seed=K + N + 1, device=DEV)
    got = abi.moe_awq_dequant_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"], dtype=torch.bfloat16)
    torch.cuda.synchronize()
    for e in range(E):
        ref = awq.dequant(_np(w["qw_gu"][e]), _np(w["qz_gu"][e]), _np(w["sc_gu"][e]), mode="bf16")
        g = f64(got[e])
        assert np.array_equal(g, ref)


def _expert_fn(w, I):
    host = {k: _np(w[k]) for k in ("qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d")}
    cache = {}

    def ew(e):
        if e not in cache:
            cache[e] = awq.expert_weights_out_in(host["qw_gu"], host["qz_gu"], host["sc_gu"], host["qw_d"],
                                                 host["qz_d"], host["sc_d"], e, I, mode="bf16")
        return cache[e]

    return ew


@pytest.mark.parametrize("T,H,I,E,k,out_fp32", [(1, 2048, 640, 512, 10, False), (8, 512, 128, 16, 4, True),
                                                (16, 1024, 192, 64, 6, False), (40, 512, 128, 16, 4, False),
                                                (300, 512, 128, 8, 3, True)])
def test_experts_awq_bf16_routed_and_shared(T, H, I, E, k, out_fp32):
    """moe_experts_awq_g32 with BF16 activations: the split-K decode kernel
    (T <= 16, plain and tile-packed weights) and the grouped GEMMs (larger
    T), routed rows and the BF16 shared expert against the oracle."""
    wl = _wl(H=H, I=I, I_sh=I, E=E, k=k)
    w = synth.make_weights(wl, seed=T + I + 5, device=DEV)
    x = synth.make_tokens(wl, T, seed=T + 5, device=DEV)
    assert x.dtype == torch.bfloat16 and w["w_sh_gate_up"].dtype == torch.bfloat16
    idx = synth.make_routing(T, E, k, seed=T + 6)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    f, sh = abi.moe_experts_awq_g32(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"],
                                    w["sc_d"], w["w_sh_gate_up"], w["w_sh_down"], out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    assert f.dtype == (torch.float32 if out_fp32 else torch.bfloat16) and sh.dtype == torch.bfloat16
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    xs = f64(x)
    ref, _ = moe.routed_outputs(xs, perm, _expert_fn(w, I))
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err < TOL_BF16, err
    sg = f64(w["w_sh_gate_up"])
    sref, _ = moe.swiglu_expert(xs, sg[:I], sg[I:], f64(w["w_sh_down"]))
    assert rel_err(f64(sh), sref) < TOL_BF16
    packed = abi.moe_awq_prepack_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"])
    fp, shp = abi.moe_experts_awq_g32_prepacked(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"],
                                                w["qz_d"], w["sc_d"], packed, w["w_sh_gate_up"], w["w_sh_down"],
                                                out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    assert torch.equal(fp, f) and torch.equal(shp, sh)


def test_grouped_swiglu_awq_bf16_prefill_shape():
    T, H, I, E, k = 700, 2048, 640, 64, 10
    wl = _wl(H=H, I=I, E=E, k=k)
    w = synth.make_weights(wl, seed=11, device=DEV)
    x = synth.make_tokens(wl, T, seed=11, device=DEV)
    idx = synth.make_routing(T, E, k, seed=12)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    f = abi.moe_grouped_swiglu_awq_g32(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"],
                                       w["sc_d"], out_fp32=True)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    ref, _ = moe.routed_outputs(f64(x), perm, _expert_fn(w, I))
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err < TOL_BF16, err


@pytest.fixture(scope="module")
def awq_bf16_layer():
    wl = synth.WORKLOADS["awq_g32_bf16"]
    return wl, synth.make_weights(wl, seed=0, device=DEV)


def _oracle(wl, w, x):
    sh = f64(w["w_sh_gate_up"])
    I = wl.I_sh
    return moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, _expert_fn(w, wl.I),
                         (sh[:I], sh[I:], f64(w["w_sh_down"])))


@pytest.mark.parametrize("T", [1, 8, 32])
def test_awq_bf16_layer_decode(awq_bf16_layer, T):
    wl, w = awq_bf16_layer
    layer = MoELayer(w, wl.k, "awq_g32", T_max=T)
    x = synth.make_tokens(wl, T, seed=2, device=DEV)
    y = layer.forward(x)
    assert y.dtype == torch.bfloat16
    ref = _oracle(wl, w, x)
    ok = ref["route"]["margin"] > 1e-3
    assert ok.any()
    assert rel_err(f64(y)[ok], ref["y"][ok]) < TOL_BF16
    assert abi.moe_device_status() == 0


def test_awq_bf16_layer_prefill_sampled(awq_bf16_layer):
    wl, w = awq_bf16_layer
    T = wl.T_prefill
    layer = MoELayer(w, wl.k, "awq_g32", T_max=T)
    x = synth.make_tokens(wl, T, seed=2, device=DEV)
    y = layer.forward(x)
    torch.cuda.synchronize()
    sample = np.concatenate([np.random.default_rng(2).choice(T, 16, replace=False), [0, T - 1]])
    ref = _oracle(wl, w, x[torch.as_tensor(sample, device=DEV)])
    ok = ref["route"]["margin"] > 1e-3
    assert rel_err(f64(y)[sample][ok], ref["y"][ok]) < TOL_BF16
    assert abi.moe_device_status() == 0
