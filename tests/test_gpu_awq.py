"""AWQ W4A16 group-32 experts on the GPU against the oracle: dequantised
weights bit for bit, grouped SwiGLU and whole layers within the 5e-2
normwise bound of the 4-bit paths (the oracle computes in float64 with its
own dequantised FP16 weights)."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from oracle import awq, moe
from tests.helpers import f64, rel_err, tile_edge_sample

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_4BIT = 5e-2


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("E,K,N", [(3, 64, 64), (2, 2048, 1280), (2, 640, 2048), (1, 96, 24)])
def test_awq_dequant_bit_exact(E, K, N):
    wl = dataclasses.replace(synth.WORKLOADS["awq_g32"], H=K, I=N // 2, E=E)
    w = synth.make_weights(wl, seed=K + N, device=DEV)
    got = abi.moe_awq_dequant_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"])
    torch.cuda.synchronize()
    for e in range(E):
        ref = awq.dequant(_np(w["qw_gu"][e]), _np(w["qz_gu"][e]), _np(w["sc_gu"][e]))
        g = _np(got[e].view(torch.int16)).view(np.uint16)
        r = ref.astype(np.float16).view(np.uint16)
        assert np.array_equal(g, r)


def _awq_expert_fn(w, I, cache: bool = True):
    store = {}
    host = {k: _np(w[k]) for k in ("qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d")}

    def ew(e):
        if e in store:
            return store[e]
        out = awq.expert_weights_out_in(host["qw_gu"], host["qz_gu"], host["sc_gu"], host["qw_d"], host["qz_d"],
                                        host["sc_d"], e, I)
        if cache:
            store[e] = out
        return out

    return ew


@pytest.mark.parametrize("T,H,I,E,k,out_fp32", [(1, 2048, 640, 512, 10, False), (2, 512, 128, 16, 4, False),
                                                (4, 256, 256, 8, 2, True), (8, 512, 128, 16, 4, True),
                                                (16, 1024, 192, 64, 6, False), (3, 256, 64, 16, 2, True),
                                                (40, 512, 128, 16, 4, False)])
def test_experts_awq_routed_and_shared(T, H, I, E, k, out_fp32):
    """moe_experts_awq_g32: routed AWQ experts (T <= 16: dequantised in the
    split-K weight-streaming kernel; larger T: the grouped AWQ GEMMs) and the
    FP16 shared expert, against the oracle."""
    wl = dataclasses.replace(synth.WORKLOADS["awq_g32"], H=H, I=I, I_sh=I, E=E, k=k)
    w = synth.make_weights(wl, seed=T + I + 3, device=DEV)
    x = synth.make_tokens(wl, T, seed=T + 3, device=DEV)
    idx = synth.make_routing(T, E, k, seed=T + 4)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    f, sh = abi.moe_experts_awq_g32(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"],
                                    w["sc_d"], w["w_sh_gate_up"], w["w_sh_down"], out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    xs = f64(x)
    ref, _ = moe.routed_outputs(xs, perm, _awq_expert_fn(w, I))
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err < 1e-2, err  # FP16 h and output rounding only
    sg = f64(w["w_sh_gate_up"])
    sref, _ = moe.swiglu_expert(xs, sg[:I], sg[I:], f64(w["w_sh_down"]))
    err_sh = rel_err(f64(sh), sref)
    assert err_sh < 1e-2, err_sh
    # the tile-packed weights give the same outputs, bit for bit (T <= 16 reads only them)
    packed = abi.moe_awq_prepack_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"])
    fp, shp = abi.moe_experts_awq_g32_prepacked(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"],
                                                w["qz_d"], w["sc_d"], packed, w["w_sh_gate_up"], w["w_sh_down"],
                                                out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    assert torch.equal(fp, f) and torch.equal(shp, sh)


def test_awq_prepack_layout():
    """Every byte of the tile-packed copy against the layout spelled out in
    numpy: per expert the gate/up units (j, kt), then the down units (j, m);
    per unit codes [r0][wc][i] (K row r0 + 16 i, code word wc), scales
    [2 groups][128 columns], zeros [2 groups][16 words]; code and zero words
    in pair order (column 2m in nibble m, column 2m + 1 in nibble m + 4)."""
    E, H, I = 3, 256, 128
    wl = dataclasses.replace(synth.WORKLOADS["awq_g32"], H=H, I=I, I_sh=I, E=E, k=2)
    w = synth.make_weights(wl, seed=7, device=DEV)
    packed = abi.moe_awq_prepack_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"])
    torch.cuda.synchronize()
    got = packed.cpu().numpy()
    h = {k: w[k].cpu().numpy() for k in ("qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d")}
    J, nka, nkb = I // 64, H // 64, H // 128
    units = []
    for e in range(E):
        for j in range(J):
            for kt in range(nka):
                words = [8 * j + c for c in range(8)] + [I // 8 + 8 * j + c for c in range(8)]
                units.append((h["qw_gu"][e], h["qz_gu"][e], h["sc_gu"][e], 64 * kt, words))
        for j in range(J):
            for m in range(nkb):
                units.append((h["qw_d"][e], h["qz_d"][e], h["sc_d"][e], 64 * j, [16 * m + c for c in range(16)]))
    def pair_order(a):
        u = a.astype(np.int64) & 0xFFFFFFFF
        o = np.zeros_like(u)
        for m in range(4):
            o |= ((u >> (8 * m)) & 0xF) << (4 * m)
            o |= ((u >> (8 * m + 4)) & 0xF) << (4 * m + 16)
        return o.astype(np.uint32).view(np.int32)

    want = []
    for qw, qz, sc, k0, words in units:
        codes = np.array([[[qw[k0 + r0 + 16 * i, words[wc]] for i in range(4)] for wc in range(16)]
                          for r0 in range(16)], dtype=np.int32)
        cols = np.array([8 * words[c // 8] + c % 8 for c in range(128)])
        scales = np.stack([sc[k0 // 32 + gi, cols] for gi in range(2)]).astype(np.float16)
        zeros = np.stack([qz[k0 // 32 + gi, words] for gi in range(2)]).astype(np.int32)
        want.append(np.concatenate([pair_order(codes).view(np.uint8).ravel(), scales.view(np.uint8).ravel(),
                                    pair_order(zeros).view(np.uint8).ravel()]))
    want = np.concatenate(want)
    assert got.size == abi.load().moe_awq_packed_bytes(E, H, I) == want.size
    assert np.array_equal(got, want)


FFN_CASES = [
    # T, H, I, E, k
    (37, 256, 64, 16, 2),
    (300, 512, 128, 8, 3),
    (1, 2048, 640, 512, 10),
    (32, 2048, 640, 512, 10),
    (700, 2048, 640, 64, 10),
]


@pytest.mark.parametrize("T,H,I,E,k", FFN_CASES)
def test_grouped_swiglu_awq(T, H, I, E, k):
    wl = dataclasses.replace(synth.WORKLOADS["awq_g32"], H=H, I=I, E=E, k=k)
    w = synth.make_weights(wl, seed=T + I, device=DEV)
    x = synth.make_tokens(wl, T, seed=T, device=DEV)
    idx = synth.make_routing(T, E, k, seed=T + 1)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    f = abi.moe_grouped_swiglu_awq_g32(x, rt, off, T * k, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"],
                                       w["sc_d"], out_fp32=True)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    ref, _ = moe.routed_outputs(f64(x), perm, _awq_expert_fn(w, I))
    g_rows = f64(f)[sr.cpu().numpy().ravel()]
    r_rows = ref[perm["slot_row"].ravel()]
    err = rel_err(g_rows, r_rows)
    assert err <= TOL_4BIT, err
    assert err < 1e-2  # FP16 h rounding only


@pytest.fixture(scope="module")
def awq_layer():
    wl = synth.WORKLOADS["awq_g32"]
    return wl, synth.make_weights(wl, seed=0, device=DEV)


def _oracle(wl, w, x):
    sh = f64(w["w_sh_gate_up"])
    I = wl.I_sh
    return moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, _awq_expert_fn(w, wl.I),
                         (sh[:I], sh[I:], f64(w["w_sh_down"])))


@pytest.mark.parametrize("T", [1, 8, 32])
def test_awq_layer_decode(awq_layer, T):
    wl, w = awq_layer
    layer = MoELayer(w, wl.k, "awq_g32", T_max=T)
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    y = layer.forward(x)
    ref = _oracle(wl, w, x)
    ok = ref["route"]["margin"] > 1e-3
    assert ok.any()
    err = rel_err(f64(y)[ok], ref["y"][ok])
    assert err <= TOL_4BIT, err


def test_awq_layer_prefill_sampled(awq_layer):
    """Full AWQ prefill batch (T=8192) as the bench runs it; at least 1024
    tokens recomputed by the oracle: every token with a row in the first or
    last 128-row tile of the three most-loaded experts, plus random ones."""
    wl, w = awq_layer
    T = wl.T_prefill
    layer = MoELayer(w, wl.k, "awq_g32", T_max=T)
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    y = layer.forward(x)
    torch.cuda.synchronize()
    r_all = moe.route(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k)
    sample = tile_edge_sample(T, moe.permute(r_all["idx"], wl.E), n_total=1024, seed=1)
    assert len(sample) >= 1024
    sh = f64(w["w_sh_gate_up"])
    ref = moe.moe_layer(f64(x)[sample], f64(w["w_router"]), f64(w["bias"]), wl.k,
                        _awq_expert_fn(w, wl.I, cache=False), (sh[:wl.I_sh], sh[wl.I_sh:], f64(w["w_sh_down"])))
    ok = ref["route"]["margin"] > 1e-3
    assert ok.mean() > 0.9
    err = rel_err(f64(y)[sample][ok], ref["y"][ok])
    assert err <= TOL_4BIT, err
    assert abi.moe_device_status() == 0
