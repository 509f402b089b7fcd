"""GPU parity of the RAZOR pruning steps: the router-norm keep statistics
(against the oracle's row norms, and the kept set against the oracle's
selection), the byte-exact slice of every per-expert tensor (against the
oracle's gather), and a pruned layer run end to end on the sliced weights
(against the oracle layer on the oracle's slices)."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from bit_expert_gemm_b200.layer import prepare_nvfp4_weights, slice_layer_weights
from oracle import moe, razor
from tests.helpers import f64, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


@pytest.mark.parametrize("E,H,act", [(16, 256, "bf16"), (512, 2048, "bf16"), (384, 2048, "f16"), (37, 72, "bf16")])
def test_router_norm_and_keep_set(E, H, act):
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], E=E, H=H, act=act)
    wr = synth.make_weights(wl, seed=E)["w_router"]
    ss, cc = abi.razor_router_norm(wr.to(DEV))
    torch.cuda.synchronize()
    w64 = f64(wr)
    n_ref = razor.router_norm(w64)
    assert np.array_equal(cc.cpu().numpy(), np.ones(E, np.int64))
    assert np.max(np.abs(np.sqrt(ss.cpu().numpy()) - n_ref) / n_ref) < 1e-12
    for keep in sorted({1, E // 2, (3 * E) // 4, E}):
        kept, ranking, score = abi.razor_select(ss, cc, keep)
        k_ref, r_ref, s_ref = razor.select_by_router_norm(w64, keep)
        srt = np.sort(s_ref)[::-1]
        gaps = np.diff(srt[::-1])[::-1]  # consecutive gaps of the descending scores
        if keep == E or gaps[keep - 1] > 1e-9 * srt[keep - 1]:
            assert np.array_equal(kept.cpu().numpy(), k_ref)
        if np.all(gaps > 1e-9 * srt[0]):
            assert np.array_equal(ranking.cpu().numpy(), r_ref)
    assert abi.moe_device_status() == 0


def _random_kept(E, keep, seed, ordered=True):
    g = torch.Generator().manual_seed(seed)
    kept = torch.randperm(E, generator=g)[:keep]
    return (kept.sort().values if ordered else kept).to(torch.int32)


SLICE_CASES = [
    # name, shape, dtype  (the leading axis is the expert index)
    ("w_gate_up bf16", (64, 256, 128), torch.bfloat16),
    ("qw_gu int32", (64, 128, 20), torch.int32),
    ("sc_d f16", (64, 5, 128), torch.float16),
    ("gs_gu f32 (8 bytes per expert)", (64, 2), torch.float32),
    ("bias f32 (4 bytes per expert)", (64,), torch.float32),
    ("sf uint8 (3 bytes per expert)", (64, 3), torch.uint8),
    ("codes uint8 (odd rows)", (64, 7, 9), torch.uint8),
]


@pytest.mark.parametrize("name,shape,dtype", SLICE_CASES)
@pytest.mark.parametrize("keep,ordered", [(32, True), (1, True), (64, True), (17, False)])
def test_slice_bit_exact(name, shape, dtype, keep, ordered):
    g = torch.Generator().manual_seed(len(name) + keep)
    raw = torch.randint(0, 256, (int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size(),),
                        generator=g, dtype=torch.uint8)
    src = raw.view(dtype).reshape(shape)
    kept = _random_kept(shape[0], keep, seed=keep, ordered=ordered)
    out = abi.razor_slice(src.to(DEV), kept.to(DEV))
    want = razor.slice_experts(src.view(torch.uint8).reshape(shape[0], -1).numpy(), kept.numpy())
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().view(torch.uint8).reshape(keep, -1).numpy(), want)
    assert abi.moe_device_status() == 0


def test_slice_full_bf16_expert_bank():
    """The Flash-Next expert bank (E=512, H=2048, I=640, BF16 gate/up and
    down, 4 GB) sliced to 256 experts: sampled experts compared byte for
    byte with the oracle's gather."""
    wl = synth.WORKLOADS["bf16"]
    w = synth.make_weights(wl, seed=0, device=DEV)
    kept = _random_kept(wl.E, 256, seed=5)
    s = slice_layer_weights(w, kept.to(DEV))
    torch.cuda.synchronize()
    assert s["w_gate_up"].shape == (256, 2 * wl.I, wl.H) and s["w_down"].shape == (256, wl.H, wl.I)
    for j in (0, 1, 77, 128, 255):
        e = int(kept[j])
        for n in ("w_gate_up", "w_down", "w_router"):
            assert torch.equal(s[n][j].cpu().view(torch.int16), w[n][e].cpu().view(torch.int16)), (n, j)
    assert np.array_equal(s["bias"].cpu().numpy(), razor.slice_experts(w["bias"].cpu().numpy(), kept.numpy()))
    assert s["w_sh_gate_up"] is w["w_sh_gate_up"]
    assert abi.moe_device_status() == 0


def test_slice_reports_out_of_range_index():
    src = torch.arange(16 * 8, dtype=torch.int32, device=DEV).reshape(16, 8)
    kept = torch.tensor([3, 16, 5], dtype=torch.int32, device=DEV)  # 16 is outside [0, E)
    out = torch.full((3, 8), -1, dtype=torch.int32, device=DEV)
    abi.razor_slice(src, kept, out=out)
    assert abi.moe_device_status(clear=True) == abi.MOE_ERR_INVALID_ARG
    o = out.cpu()
    assert torch.equal(o[0], src[3].cpu()) and torch.equal(o[2], src[5].cpu()) and bool((o[1] == -1).all())
    assert abi.moe_device_status() == 0


@pytest.mark.parametrize("fmt", ["bf16", "awq_g32", "nvfp4"])
def test_pruned_layer_forward(fmt):
    """A layer pruned to half its experts on the GPU (router rows, bias and
    every expert tensor of the format sliced with one kept list) against the
    oracle layer on the oracle's slices of the same tensors.  The kept list
    is the oracle's router-norm selection."""
    base = {"bf16": synth.WORKLOADS["tiny"], "awq_g32": synth.WORKLOADS["awq_g32"],
            "nvfp4": synth.WORKLOADS["nvfp4"]}[fmt]
    wl = dataclasses.replace(base, H=256, I=128, I_sh=128, E=32, k=4)
    T = 96
    w = synth.make_weights(wl, seed=3, device=DEV)
    if fmt == "nvfp4":
        w = prepare_nvfp4_weights(w)
    x = synth.make_tokens(wl, T, seed=3, device=DEV)
    keep = wl.E // 2
    k_ref, _, _ = razor.select_by_router_norm(f64(w["w_router"]), keep)
    ws = slice_layer_weights(w, torch.from_numpy(k_ref.astype(np.int32)).to(DEV))
    layer = MoELayer(ws, wl.k, fmt, T_max=T)
    assert layer.E == keep
    y = f64(layer.forward(x))
    # oracle: slice the inputs on the host, then the plain layer
    hk = lambda n: razor.slice_experts(w[n].cpu().numpy(), k_ref)  # noqa: E731
    xs = f64(x)
    wr_s = razor.slice_experts(f64(w["w_router"]), k_ref)
    r = moe.route(xs, wr_s, hk("bias").astype(np.float64), wl.k)
    p = moe.permute(r["idx"], keep)
    sh, _ = moe.swiglu_expert(xs, *shared_fn(w))
    if fmt == "bf16":
        gu = f64(w["w_gate_up"])[k_ref]
        wd = f64(w["w_down"])[k_ref]
        f, _ = moe.routed_outputs(xs, p, lambda e: (gu[e, :wl.I], gu[e, wl.I:], wd[e]))
        tol = TOL_BF16
    elif fmt == "awq_g32":
        from oracle import awq as oawq

        q = {n: hk(n) for n in ("qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d")}
        f, _ = moe.routed_outputs(xs, p, lambda e: oawq.expert_weights_out_in(
            q["qw_gu"], q["qz_gu"], q["sc_gu"], q["qw_d"], q["qz_d"], q["sc_d"], e, wl.I))
        tol = 5e-2
    else:
        from oracle import nvfp4 as onv

        deq, _ = onv.quantize_expert_weights(f64(w["w_gate_up"])[k_ref], f64(w["w_down"])[k_ref])
        f, _, _ = onv.routed_outputs_w4a4(xs, p, deq)
        tol = 5e-2
    y_ref = moe.combine(f, p["slot_row"], r["w"], sh)
    ok = r["margin"] > 1e-3
    assert ok.mean() > 0.8
    assert np.array_equal(layer.topk_idx[:T].cpu().numpy()[ok], r["idx"][ok])
    assert rel_err(y[ok], y_ref[ok]) < tol
    assert abi.moe_device_status() == 0
