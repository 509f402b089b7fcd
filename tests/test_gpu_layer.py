"""Whole-layer GPU parity: the MoE forward (route -> permute -> grouped
SwiGLU -> shared expert -> combine) and the Refill-RMS pass, run through the
C ABI by MoELayer, against the CPU oracle.  Outputs are compared on the
tokens whose routing is decided by a logit margin above 1e-3 (the others may
legitimately pick different experts in FP32 than in FP64)."""

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from oracle import moe, razor
from tests.helpers import expert_fn_bf16, f64, refill_stats_ref, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def bf16_layer():
    wl = synth.WORKLOADS["bf16"]
    w = synth.make_weights(wl, seed=0, device=DEV)
    return wl, w


def _oracle_tokens(wl, w, x, extra=0):
    return moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, expert_fn_bf16(w, wl.I), shared_fn(w),
                         extra=extra)


def test_tiny_layer_forward():
    wl = synth.WORKLOADS["tiny"]
    w = {n: t.to(DEV) for n, t in synth.make_weights(wl, seed=0).items()}
    x = synth.make_tokens(wl, wl.T_prefill, seed=0).to(DEV)
    layer = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill)
    y = layer.forward(x)
    ref = _oracle_tokens(wl, w, x)
    ok = ref["route"]["margin"] > 1e-3
    assert ok.mean() > 0.8
    err = rel_err(f64(y)[ok], ref["y"][ok])
    assert err <= TOL_BF16, err
    assert abi.moe_device_status() == 0


@pytest.mark.parametrize("T,graphs", [(64, True), (1, True), (8, False), (300, True)])
def test_host_pipeline_matches_forward(bf16_layer, T, graphs):
    """Batches streamed from pinned host memory by HostPipeline (decode
    sizes: one graph per step with the copies inside; larger batches: uploads
    and downloads overlapped with the neighbouring forwards) come back bit for
    bit equal to the device forward of the same batches, including when more
    batches than buffers are in flight."""
    from bit_expert_gemm_b200.layer import HostPipeline
    wl, w = bf16_layer
    layer = MoELayer(w, wl.k, "bf16", T_max=T)
    xs = [synth.make_tokens(wl, T, seed=s, device=DEV) for s in range(5)]
    want = [layer.forward(x).clone() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty((T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in xs]
    pipe = HostPipeline(layer, T, use_graphs=graphs)
    pipe.begin()
    for i in range(len(xs)):
        pipe.step(xh[i], yh[i])
    pipe.finish()
    torch.cuda.synchronize()
    for i in range(len(xs)):
        assert torch.equal(yh[i], want[i].cpu()), i
    assert abi.moe_device_status() == 0


@pytest.mark.parametrize("T", [1, 8, 64])
def test_bf16_layer_decode(bf16_layer, T):
    wl, w = bf16_layer
    layer = MoELayer(w, wl.k, "bf16", T_max=T)
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    y = layer.forward(x)
    ref = _oracle_tokens(wl, w, x)
    ok = ref["route"]["margin"] > 1e-3
    assert ok.any()
    err = rel_err(f64(y)[ok], ref["y"][ok])
    assert err <= TOL_BF16, err


def test_bf16_layer_prefill_sampled(bf16_layer):
    """Full prefill batch (T=8192) in the launch configuration the bench
    times; 24 sampled tokens recomputed one by one by the oracle (the layer
    is per-token, so a subset is exact)."""
    wl, w = bf16_layer
    T = wl.T_prefill
    layer = MoELayer(w, wl.k, "bf16", T_max=T)
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    y = layer.forward(x)
    torch.cuda.synchronize()
    sample = np.random.default_rng(0).choice(T, 24, replace=False)
    sample = np.concatenate([sample, [0, T - 1]])
    ref = _oracle_tokens(wl, w, x[torch.as_tensor(sample, device=DEV)])
    ok = ref["route"]["margin"] > 1e-3
    err = rel_err(f64(y)[sample][ok], ref["y"][ok])
    assert err <= TOL_BF16, err
    # properties that hold at any size: a valid permutation of all T*k assignments
    off = layer.offsets.cpu().numpy()
    assert off[0] == 0 and off[-1] == T * wl.k and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.sort(layer.slot_row[:T].cpu().numpy().ravel()), np.arange(T * wl.k))
    assert abi.moe_device_status() == 0


def test_tiny_refill_pass_and_selection():
    wl = synth.WORKLOADS["tiny"]
    w = {n: t.to(DEV) for n, t in synth.make_weights(wl, seed=0).items()}
    x = synth.make_tokens(wl, wl.T_prefill, seed=0).to(DEV)
    layer = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill, extra=1)
    ss = torch.zeros(wl.E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=DEV)
    y = layer.refill_pass(x, ss, cc)
    ref = _oracle_tokens(wl, w, x, extra=1)
    s_ref, c_ref, good = refill_stats_ref(ref, wl.k, wl.E)
    assert len(good) >= wl.E // 2
    assert np.array_equal(cc.cpu().numpy()[good], c_ref[good])
    assert rel_err(ss.cpu().numpy()[good], s_ref[good]) < TOL_BF16
    ok = ref["route"]["margin"] > 1e-3
    assert rel_err(f64(y)[ok], ref["y"][ok]) < TOL_BF16
    if len(good) == wl.E:
        keep = wl.E // 2
        kept, _, _ = abi.razor_select(ss, cc, keep)
        k_ref, _, sc = razor.select(s_ref, c_ref, keep)
        srt = np.sort(sc)[::-1]
        if srt[keep - 1] - srt[keep] > 4 * TOL_BF16 * srt[keep - 1]:
            assert np.array_equal(kept.cpu().numpy(), k_ref)


def test_refill_full_row_additive_and_sampled(bf16_layer):
    """One packed row of T=32768 tokens (the Refill workload) in the bench's
    launch configuration: statistics are additive (full pass == sum of four
    chunk passes), every selected assignment is counted once, and a sampled
    chunk matches the oracle."""
    wl, w = bf16_layer
    T = synth.WORKLOADS["refill"].T_prefill
    x = synth.make_tokens(synth.WORKLOADS["refill"], T, seed=0, device=DEV)
    layer = MoELayer(w, wl.k, "bf16", T_max=T, extra=1)
    ss = torch.zeros(wl.E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=DEV)
    layer.refill_pass(x, ss, cc)
    ss4 = torch.zeros_like(ss)
    cc4 = torch.zeros_like(cc)
    for a in range(0, T, T // 4):
        layer.refill_pass(x[a:a + T // 4], ss4, cc4)
    torch.cuda.synchronize()
    assert int(cc.sum()) == T * wl.k
    assert torch.equal(cc, cc4)
    assert rel_err(ss4.cpu().numpy(), ss.cpu().numpy()) < 1e-9
    # sampled chunk against the oracle
    n = 48
    xs = x[1000:1000 + n]
    ss_s = torch.zeros_like(ss)
    cc_s = torch.zeros_like(cc)
    layer.refill_pass(xs, ss_s, cc_s)
    ref = _oracle_tokens(wl, w, xs, extra=1)
    s_ref, c_ref, good = refill_stats_ref(ref, wl.k, wl.E)
    assert np.array_equal(cc_s.cpu().numpy()[good], c_ref[good])
    assert rel_err(ss_s.cpu().numpy()[good], s_ref[good]) < TOL_BF16
