"""The pre-MoE RMSNorm and the shared-expert gate in the layer's forward
(moe_norm_route_permute: one cooperative kernel for T <= 128, the norm
kernel then the large-batch routing above), against the oracle: the block
input x_norm within one 16-bit step of the oracle's BF16-rounded norm,
the gate, the routing of decided tokens bit for bit, and the layer output
within the BF16 bound."""

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from oracle import moe
from tests.helpers import expert_fn_bf16, f64, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


def _weights(wl, seed):
    w = synth.make_weights(wl, seed=seed, device=DEV)
    w["w_norm"] = synth.make_norm_weight(wl, seed, device=DEV)
    w["w_sh_gate"] = synth.make_shared_gate(wl, seed, device=DEV)
    return w


def _oracle(wl, w, x):
    xin = moe.block_input(f64(x), f64(w["w_norm"]), 1e-6)
    out = moe.moe_layer(xin, f64(w["w_router"]), f64(w["bias"]), wl.k, expert_fn_bf16(w, wl.I, cache=False),
                        shared_fn(w), shared_gate_w=f64(w["w_sh_gate"]))
    out["xin"] = xin
    out["gate"] = moe.shared_gate(xin, f64(w["w_sh_gate"]))
    return out


def _decided_tokens(wl, w, T, seed):
    """A token batch of size T whose oracle routing is decided for most
    tokens (for T = 1: the first seed from `seed` on whose one token is)."""
    for s in range(seed, seed + 50):
        x = synth.make_tokens(wl, T, seed=s, device=DEV)
        xin = moe.block_input(f64(x), f64(w["w_norm"]), 1e-6)
        if (moe.route(xin, f64(w["w_router"]), f64(w["bias"]), wl.k)["margin"] > 1e-3).mean() > 0.8:
            return x
    raise AssertionError("no decided batch")


def _check(wl, w, T, seed):
    x = _decided_tokens(wl, w, T, seed)
    layer = MoELayer(w, wl.k, "bf16", T_max=T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    ref = _oracle(wl, w, x)
    xn = f64(layer.x_norm[:T])
    # one 16-bit step at most (the FP32 norm rounds once to BF16; the oracle's
    # exact norm rounds once from float64), and nearly always equal
    step = np.ldexp(1.0, np.frexp(ref["xin"])[1] - 8)
    assert np.all(np.abs(xn - ref["xin"]) <= step)
    assert np.mean(xn == ref["xin"]) > 0.999
    assert np.max(np.abs(f64(layer.sh_gate[:T]) - ref["gate"])) < 1e-4
    ok = ref["route"]["margin"] > 1e-3
    assert ok.mean() > 0.8
    assert np.array_equal(layer.topk_idx[:T].cpu().numpy()[ok], ref["route"]["idx"][ok])
    err = rel_err(f64(y)[ok], ref["y"][ok])
    assert err <= TOL_BF16, err
    return layer, x


def test_tiny_layer_with_norm_and_gate():
    wl = synth.WORKLOADS["tiny"]
    _check(wl, _weights(wl, 0), wl.T_prefill, 0)


@pytest.mark.parametrize("T", [1, 8, 64, 512])
def test_bf16_layer_with_norm_and_gate(T):
    """T <= 128: norm, gate, logits, top-k and permutation in the one
    cooperative kernel; T = 512: the norm kernel, then the router GEMM."""
    wl = synth.WORKLOADS["bf16"]
    layer, x = _check(wl, _weights(wl, 1), T, 3)
    # the fused routing equals the plain routing of the x_norm it produced
    idx, w_, _, off, rt, sr = abi.moe_route_permute(layer.x_norm[:T].clone(), layer.w["w_router"], layer.w["bias"],
                                                    wl.k)
    torch.cuda.synchronize()
    assert torch.equal(idx, layer.topk_idx[:T]) and torch.equal(off, layer.offsets)
    assert torch.equal(rt, layer.row_token[:T * wl.k]) and torch.equal(w_, layer.topk_w[:T])


def test_norm_paths_agree_on_x_norm():
    """The block-per-token norm of the cooperative kernel and the
    warp-per-token norm kernel sum the squares in different orders: their
    x_norm differ at most by one 16-bit step, rarely."""
    wl = synth.WORKLOADS["bf16"]
    w = _weights(wl, 2)
    x = synth.make_tokens(wl, 96, seed=5, device=DEV)
    a = abi.moe_norm_route_permute(x, w["w_norm"], w["w_router"], w["bias"], wl.k, w_shared_gate=w["w_sh_gate"])
    b = abi.moe_rmsnorm(x, w["w_norm"])
    g = abi.moe_shared_gate(b, w["w_sh_gate"])
    torch.cuda.synchronize()
    xa, xb = f64(a[0]), f64(b)
    step = np.ldexp(1.0, np.frexp(xb)[1] - 8)
    assert np.all(np.abs(xa - xb) <= step) and np.mean(xa == xb) > 0.999
    assert torch.allclose(a[1], g, rtol=0, atol=1e-5)
