"""GPU parity of each C-ABI operation against the CPU oracle, element by
element on seeded inputs.  Integer outputs (routing indices where the logit
margin exceeds 1e-3, permutations, kept sets, rankings) must match bit for
bit; floating-point outputs must stay within the normwise relative error
max|gpu - oracle| / max|oracle| <= 2e-2 that BF16 outputs are held to."""

import dataclasses

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import abi, synth
from oracle import moe, razor
from tests.helpers import f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


def _wl(**kw):
    return dataclasses.replace(synth.WORKLOADS["tiny"], **kw)


@pytest.mark.parametrize("T,E,ks", [(0, 16, 2), (1, 512, 10), (7, 16, 2), (64, 512, 10), (1000, 512, 11),
                                    (4099, 64, 3), (8192, 512, 10), (33, 1024, 16)])
def test_permute_bit_exact(T, E, ks):
    idx = synth.make_routing(max(T, 1), E, ks, seed=T + E)[:T].contiguous()
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    want = moe.permute(idx.numpy().astype(np.int64), E)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy(), want["offsets"])
    assert np.array_equal(rt.cpu().numpy(), want["row_token"])
    assert np.array_equal(sr.cpu().numpy(), want["slot_row"])
    assert abi.moe_device_status() == 0


def test_permute_reports_out_of_range_index():
    idx = synth.make_routing(16, 16, 2, seed=1).clone()
    idx[3, 1] = 16  # outside [0, E)
    abi.moe_permute(idx.to(DEV), 16)
    assert abi.moe_device_status(clear=True) == abi.MOE_ERR_INVALID_ARG
    assert abi.moe_device_status() == 0


ROUTE_CASES = [
    # T, H, E, k, extra, bias_std, act  (T >= 256 and E % 64 == 0 take the tensor-core logits path)
    (64, 256, 16, 2, 0, 1.0, "bf16"),
    (64, 256, 16, 2, 1, 1.0, "bf16"),
    (1, 2048, 512, 10, 0, 1.5, "bf16"),
    (64, 2048, 512, 10, 1, 1.5, "bf16"),
    (1024, 2048, 512, 10, 0, 1.5, "bf16"),
    (300, 512, 384, 10, 1, 1.5, "bf16"),
    (520, 2048, 512, 10, 0, 1.5, "f16"),
    (32, 2048, 512, 10, 0, 1.5, "f16"),
]


@pytest.mark.parametrize("T,H,E,k,extra,bstd,act", ROUTE_CASES)
def test_route_topk(T, H, E, k, extra, bstd, act):
    wl = _wl(H=H, E=E, k=k, bias_std=bstd, act=act)
    w = synth.make_weights(wl, seed=3, device=DEV)
    x = synth.make_tokens(wl, T, seed=3, device=DEV)
    idx, wt, lg = abi.moe_route_topk(x, w["w_router"], w["bias"], k, extra)
    r = moe.route(f64(x), f64(w["w_router"]), f64(w["bias"]), k, extra)
    ok = r["margin"] > 1e-3
    assert ok.mean() > 0.8
    gi = idx.cpu().numpy()
    assert np.array_equal(gi[ok], r["idx"][ok])
    assert np.allclose(wt.cpu().numpy()[ok], r["w"][ok], atol=2e-5, rtol=1e-4)
    want_logit = np.take_along_axis(r["logits"], gi.astype(np.int64), 1)
    assert np.allclose(lg.cpu().numpy(), want_logit, atol=2e-3, rtol=1e-4)
    assert np.allclose(wt.cpu().numpy().sum(1), 1.0, atol=1e-5)


def _ffn_case(T, H, I, E, k, act, seed):
    wl = _wl(H=H, I=I, E=E, k=k, act=act)
    w = synth.make_weights(wl, seed=seed, device=DEV)
    if act == "f16":  # 16-bit expert weights follow the activation dtype
        w["w_gate_up"] = w["w_gate_up"].to(torch.float16)
        w["w_down"] = w["w_down"].to(torch.float16)
    x = synth.make_tokens(wl, T, seed=seed, device=DEV)
    idx = synth.make_routing(T, E, k, seed=seed)
    return wl, w, x, idx


FFN_CASES = [
    # T, H, I, E, k, act, out_fp32
    (37, 256, 64, 16, 2, "bf16", False),
    (300, 512, 128, 8, 3, "bf16", False),
    (2000, 1024, 256, 32, 4, "bf16", True),
    (1, 2048, 640, 512, 10, "bf16", False),
    (64, 2048, 640, 512, 10, "bf16", False),
    (700, 2048, 640, 64, 10, "bf16", False),
    (129, 512, 192, 5, 2, "f16", False),
]


@pytest.mark.parametrize("T,H,I,E,k,act,out_fp32", FFN_CASES)
def test_grouped_swiglu_16bit(T, H, I, E, k, act, out_fp32):
    wl, w, x, idx = _ffn_case(T, H, I, E, k, act, seed=T + I)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    rows = T * k
    f = abi.moe_grouped_swiglu_bf16(x, rt, off, rows, w["w_gate_up"], w["w_down"], out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    xs = f64(x)
    gu, wd = w["w_gate_up"], w["w_down"]
    ref, _ = moe.routed_outputs(xs, perm, lambda e: (f64(gu[e, :I]), f64(gu[e, I:]), f64(wd[e])))
    got = f64(f)
    gsr = sr.cpu().numpy()
    g_rows = got[gsr.ravel()]
    r_rows = ref[perm["slot_row"].ravel()]
    err = rel_err(g_rows, r_rows)
    assert err <= TOL_BF16, err
    assert err < 1e-2


def test_dense_expert_identity_rows():
    wl, w, x, _ = _ffn_case(300, 512, 128, 1, 1, "bf16", seed=5)
    off = torch.tensor([0, 300], dtype=torch.int32, device=DEV)
    f = abi.moe_grouped_swiglu_bf16(x, None, off, 300, w["w_sh_gate_up"].unsqueeze(0), w["w_sh_down"].unsqueeze(0))
    sg = f64(w["w_sh_gate_up"])
    ref, _ = moe.swiglu_expert(f64(x), sg[:64], sg[64:], f64(w["w_sh_down"]))
    assert rel_err(f64(f), ref) < 1e-2


@pytest.mark.parametrize("T,H,I,act,out_fp32", [(1, 2048, 640, "bf16", False), (3, 2048, 640, "f16", True),
                                               (8, 256, 64, "bf16", False), (16, 2560, 640, "bf16", True),
                                               (13, 512, 128, "f16", False)])
def test_dense_expert_decode_gemv(T, H, I, act, out_fp32):
    """One dense expert (the shared expert) on a decode batch: the
    weight-streaming GEMV path of moe_grouped_swiglu_bf16, against the
    oracle; an expert row range that ends before the batch leaves the later
    output rows untouched."""
    wl, w, x, _ = _ffn_case(T, H, I, 1, 1, act, seed=T + 21)
    gu, wd = w["w_gate_up"][0], w["w_down"][0]  # expert 0 as the dense expert
    sg = f64(gu)
    ref, _ = moe.swiglu_expert(f64(x), sg[:I], sg[I:], f64(wd))
    off = torch.tensor([0, T], dtype=torch.int32, device=DEV)
    f = abi.moe_grouped_swiglu_bf16(x, None, off, T, gu.unsqueeze(0), wd.unsqueeze(0), out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    assert rel_err(f64(f), ref) < TOL_BF16
    if T > 2:
        off2 = torch.tensor([0, T - 2], dtype=torch.int32, device=DEV)
        f2 = torch.full_like(f, 7.0)
        abi.moe_grouped_swiglu_bf16(x, None, off2, T, gu.unsqueeze(0), wd.unsqueeze(0), out_fp32=out_fp32, f=f2)
        torch.cuda.synchronize()
        assert torch.equal(f2[: T - 2], f[: T - 2]) and bool((f2[T - 2:] == 7.0).all())


@pytest.mark.parametrize("T,H,E,k,ks,f32", [(1, 2048, 512, 10, 10, False), (300, 512, 16, 3, 4, False),
                                            (257, 2048, 64, 10, 11, True)])
def test_combine(T, H, E, k, ks, f32):
    idx = synth.make_routing(T, E, ks, seed=T)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    wl = _wl(H=H)
    f = synth.make_tokens(wl, T * ks, seed=11, device=DEV)
    if f32:
        f = f.float() * 3
    shared = synth.make_tokens(wl, T, seed=12, device=DEV)
    wt = synth.make_weights_topk(T, k, seed=T).to(DEV)
    y = abi.moe_combine(f, sr, wt, shared_out=shared)
    ref = moe.combine(f64(f), sr.cpu().numpy(), wt.double().cpu().numpy(), f64(shared))
    assert rel_err(f64(y), ref) < 1e-2


@pytest.mark.parametrize("E", [1, 16, 256, 512, 1000, 1024])
def test_select_bit_exact(E):
    for seed in range(3):
        ss, cc = synth.make_refill_stats(E, seed)
        for keep in sorted({0, 1, E // 2, min(E, 256), E}):
            kept, ranking, score = abi.razor_select(ss.to(DEV), cc.to(DEV), keep)
            k_ref, r_ref, s_ref = razor.select(ss.numpy(), cc.numpy(), keep)
            assert np.array_equal(score.cpu().numpy(), s_ref)
            assert np.array_equal(ranking.cpu().numpy(), r_ref)
            assert np.array_equal(kept.cpu().numpy(), k_ref)


@pytest.mark.parametrize("T,H,I,E,k,out_fp32,act", [
    # T <= 16: one split-K kernel + partial sums
    (1, 2048, 640, 512, 10, False, "bf16"), (2, 512, 128, 16, 4, True, "bf16"), (4, 256, 256, 16, 3, False, "f16"),
    (3, 512, 384, 32, 2, False, "bf16"), (8, 512, 128, 16, 4, False, "bf16"), (3, 256, 64, 16, 2, False, "bf16"),
    (16, 1024, 192, 64, 6, True, "bf16"), (5, 384, 128, 32, 4, False, "f16"),
    # the split-K kernel at its widest H (28 blocks of 128 rows in TMEM) and at the fact sheet's 2560;
    # above 3584 the two weight-streaming GEMMs serve T <= 16 too
    (4, 3584, 256, 16, 4, True, "bf16"), (1, 2560, 640, 64, 10, False, "bf16"), (2, 4096, 128, 16, 3, False, "f16"),
    # 16 < T <= 128: two weight-streaming GEMMs
    (17, 512, 128, 16, 3, False, "bf16"), (64, 2048, 640, 64, 10, True, "bf16"), (128, 256, 64, 16, 2, False, "bf16"),
    # T > 128: the grouped prefill GEMMs
    (300, 512, 128, 8, 3, False, "bf16")])
def test_experts_routed_and_shared(T, H, I, E, k, out_fp32, act):
    """moe_experts_bf16 on all three of its paths, routed rows and the shared
    expert against the oracle."""
    wl = _wl(H=H, I=I, I_sh=I, E=E, k=k, act=act)
    w = synth.make_weights(wl, seed=T + 7, device=DEV)
    if act == "f16":
        for key in ("w_gate_up", "w_down", "w_sh_gate_up", "w_sh_down"):
            w[key] = w[key].to(torch.float16)
    x = synth.make_tokens(wl, T, seed=T + 7, device=DEV)
    idx = synth.make_routing(T, E, k, seed=T + 8)
    off, rt, sr = abi.moe_permute(idx.to(DEV), E)
    f, sh = abi.moe_experts_bf16(x, rt, off, T * k, w["w_gate_up"], w["w_down"], w["w_sh_gate_up"], w["w_sh_down"],
                                 out_fp32=out_fp32)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    perm = moe.permute(idx.numpy().astype(np.int64), E)
    xs = f64(x)
    gu, wd = w["w_gate_up"], w["w_down"]
    ref, _ = moe.routed_outputs(xs, perm, lambda e: (f64(gu[e, :I]), f64(gu[e, I:]), f64(wd[e])))
    err = rel_err(f64(f)[sr.cpu().numpy().ravel()], ref[perm["slot_row"].ravel()])
    assert err < 1e-2, err
    sg = f64(w["w_sh_gate_up"])
    sref, _ = moe.swiglu_expert(xs, sg[:I], sg[I:], f64(w["w_sh_down"]))
    err_sh = rel_err(f64(sh), sref)
    assert err_sh < 1e-2, err_sh


ROUTE_PERMUTE_CASES = [
    # T, H, E, k, extra, bias_std, act  (T <= 128: one cooperative kernel; T > 128: route then permute)
    (1, 2048, 512, 10, 0, 1.5, "bf16"),
    (7, 256, 16, 2, 0, 1.0, "bf16"),
    (33, 512, 64, 4, 1, 1.0, "f16"),
    (64, 2048, 512, 10, 1, 1.5, "bf16"),
    (128, 2048, 512, 10, 0, 1.5, "bf16"),
    (100, 256, 1000, 15, 1, 5.0, "bf16"),  # wide bias spread: 16 of 1000 still separates
    (129, 512, 384, 10, 0, 1.5, "bf16"),
    (300, 2048, 512, 10, 0, 1.5, "bf16"),
]


def _check_permutation_valid(gi, off, rt, sr, E):
    """The permutation is a function of the selection: check it against the
    selection it was built from (expert blocks ascending, tokens ascending
    inside a block, every assignment's row pointing back at its token)."""
    T, ks = gi.shape
    counts = np.bincount(gi.ravel(), minlength=E) if T else np.zeros(E, np.int64)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    for t in range(T):
        for j in range(ks):
            r = sr[t, j]
            e = gi[t, j]
            assert off[e] <= r < off[e + 1] and rt[r] == t
    for e in range(E):
        blk = rt[off[e]:off[e + 1]]
        assert np.all(np.diff(blk) > 0)


@pytest.mark.parametrize("T,H,E,k,extra,bstd,act", ROUTE_PERMUTE_CASES)
def test_route_permute(T, H, E, k, extra, bstd, act):
    wl = _wl(H=H, E=E, k=k, bias_std=bstd, act=act)
    w = synth.make_weights(wl, seed=5, device=DEV)
    x = synth.make_tokens(wl, T, seed=5, device=DEV)
    idx, wt, lg, off, rt, sr = abi.moe_route_permute(x, w["w_router"], w["bias"], k, extra)
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    r = moe.route(f64(x), f64(w["w_router"]), f64(w["bias"]), k, extra)
    ok = r["margin"] > 1e-3
    gi = idx.cpu().numpy()
    assert ok.mean() > 0.8
    assert np.array_equal(gi[ok], r["idx"][ok])
    assert np.allclose(wt.cpu().numpy()[ok], r["w"][ok], atol=2e-5, rtol=1e-4)
    want_logit = np.take_along_axis(r["logits"], gi.astype(np.int64), 1)
    assert np.allclose(lg.cpu().numpy(), want_logit, atol=2e-3, rtol=1e-4)
    off_n, rt_n, sr_n = off.cpu().numpy(), rt.cpu().numpy(), sr.cpu().numpy()
    _check_permutation_valid(gi, off_n, rt_n, sr_n, E)
    if ok.all():  # the selection is unique: so is the permutation
        want = moe.permute(r["idx"].astype(np.int64), E)
        assert np.array_equal(off_n, want["offsets"])
        assert np.array_equal(rt_n, want["row_token"])
        assert np.array_equal(sr_n, want["slot_row"])


def test_route_permute_empty_batch():
    wl = _wl(H=256, E=16, k=2)
    w = synth.make_weights(wl, seed=1, device=DEV)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    off = torch.full((17,), -7, dtype=torch.int32, device=DEV)
    abi.moe_route_permute(x, w["w_router"], w["bias"], 2, expert_offsets=off)
    torch.cuda.synchronize()
    assert off.cpu().tolist() == [0] * 17


@pytest.mark.parametrize("T,H,act", [(1, 2048, "bf16"), (64, 256, "bf16"), (777, 2048, "f16"), (8192, 2048, "bf16"),
                                     (5, 72, "bf16")])
def test_shared_gate(T, H, act):
    wl = _wl(H=H, act=act)
    x = synth.make_tokens(wl, T, seed=T)
    g = synth.make_shared_gate(wl, seed=T)
    got = abi.moe_shared_gate(x.to(DEV), g.to(DEV))
    want = moe.shared_gate(f64(x), f64(g))
    torch.cuda.synchronize()
    # FP32 dot products of H terms; the gate's slope is at most 1/4
    assert np.max(np.abs(got.cpu().double().numpy() - want)) < 1e-5
    assert abi.moe_device_status() == 0


def test_layer_with_shared_gate_forward_and_refill():
    from bit_expert_gemm_b200 import MoELayer
    from tests.helpers import expert_fn_bf16, refill_stats_ref, shared_fn

    wl = synth.WORKLOADS["tiny"]
    w = synth.make_weights(wl, seed=6, device=DEV)
    w["w_sh_gate"] = synth.make_shared_gate(wl, seed=6, device=DEV)
    x = synth.make_tokens(wl, wl.T_prefill, seed=6, device=DEV)
    ref = moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, expert_fn_bf16(w, wl.I), shared_fn(w),
                        shared_gate_w=f64(w["w_sh_gate"]))
    ok = ref["route"]["margin"] > 1e-3
    y = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill).forward(x)
    assert rel_err(f64(y)[ok], ref["y"][ok]) < TOL_BF16
    rl = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill, extra=1)
    ss = torch.zeros(wl.E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=DEV)
    y2 = rl.refill_pass(x, ss, cc)
    assert rel_err(f64(y2)[ok], ref["y"][ok]) < TOL_BF16
    ref1 = moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, expert_fn_bf16(w, wl.I), shared_fn(w),
                         extra=1)
    s_ref, c_ref, good = refill_stats_ref(ref1, wl.k, wl.E)  # the gate does not change the scores
    assert np.array_equal(cc.cpu().numpy()[good], c_ref[good])
    assert rel_err(ss.cpu().numpy()[good], s_ref[good]) < TOL_BF16
    assert abi.moe_device_status() == 0


@pytest.mark.parametrize("T,H,act,inplace", [(1, 2048, "bf16", False), (7, 256, "f16", True),
                                             (8192, 2048, "bf16", False), (33, 2560, "bf16", True)])
def test_rmsnorm(T, H, act, inplace):
    wl = _wl(H=H, act=act)
    x = synth.make_tokens(wl, T, seed=T + 3, device=DEV)
    g = synth.make_shared_gate(wl, seed=T + 3, device=DEV)  # any [H] vector serves as the gain w
    want = moe.rmsnorm(f64(x), f64(g))
    y = abi.moe_rmsnorm(x, g, y=x if inplace else None)
    torch.cuda.synchronize()
    assert (y.data_ptr() == x.data_ptr()) == inplace
    # FP32 sums, one rounding to 16 bits
    assert rel_err(f64(y), want) < 1e-2
    assert abi.moe_device_status() == 0
