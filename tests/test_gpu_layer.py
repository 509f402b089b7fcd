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
from tests.helpers import expert_fn_bf16, f64, kept_set_swaps, rel_err, shared_fn, tile_edge_sample

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
    times.  The layer is per token, so a sample of tokens recomputed by the
    oracle is exact: every token with a row in the first or last 128-row
    tile of the three most-loaded experts (the tile edges of the longest
    groups), plus random tokens, at least 1024 in all."""
    wl, w = bf16_layer
    T = wl.T_prefill
    layer = MoELayer(w, wl.k, "bf16", T_max=T)
    x = synth.make_tokens(wl, T, seed=0, device=DEV)
    y = layer.forward(x)
    torch.cuda.synchronize()
    r_all = moe.route(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k)
    sample = tile_edge_sample(T, moe.permute(r_all["idx"], wl.E), n_total=1024, seed=0)
    assert len(sample) >= 1024
    ref = moe.moe_layer(f64(x)[sample], f64(w["w_router"]), f64(w["bias"]), wl.k,
                        expert_fn_bf16(w, wl.I, cache=False), shared_fn(w))
    ok = ref["route"]["margin"] > 1e-3
    assert ok.mean() > 0.9
    err = rel_err(f64(y)[sample][ok], ref["y"][ok])
    assert err <= TOL_BF16, err
    # properties that hold at any size: a valid permutation of all T*k assignments
    off = layer.offsets.cpu().numpy()
    assert off[0] == 0 and off[-1] == T * wl.k and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.sort(layer.slot_row[:T].cpu().numpy().ravel()), np.arange(T * wl.k))
    # the routing of every decided token equals the oracle's, bit for bit
    dec = r_all["margin"] > 1e-3
    assert np.array_equal(layer.topk_idx[:T].cpu().numpy()[dec], r_all["idx"][dec])
    assert abi.moe_device_status() == 0


def _refill_oracle_stats(r, perm, f, k, E, tokens, chunk=2048):
    """Oracle Refill statistics (closed form, pinned to the definition and to
    knock-out re-evaluation) accumulated over the given tokens."""
    s = np.zeros(E)
    c = np.zeros(E, np.int64)
    for a in range(0, len(tokens), chunk):
        tk = tokens[a:a + chunk]
        d = razor.refill_deltas_closed_form(f, perm["slot_row"][tk], r["idx"][tk], r["p"][tk], k)
        razor.accumulate(s, c, d, r["idx"][tk], k)
    return s, c


def _check_refill_stats(layer, x, r, perm, f, k, E, keep, tokens):
    """GPU Refill pass over x[tokens] against the oracle's statistics over
    the same tokens (whose selections, rank k+1 included, are decided):
    counts bit-exact for every expert, sums of squares within 2e-2 of each
    expert's, and the kept set exact except swaps inside the tolerance band
    at the keep boundary.  Returns the swaps."""
    ss = torch.zeros(E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(E, dtype=torch.int64, device=DEV)
    layer.refill_pass(x[torch.as_tensor(tokens, device=DEV)], ss, cc)
    s_ref, c_ref = _refill_oracle_stats(r, perm, f, k, E, tokens)
    assert np.array_equal(cc.cpu().numpy(), c_ref)
    hit = c_ref > 0
    s_gpu = ss.cpu().numpy()
    assert np.all(s_gpu[~hit] == 0)
    assert np.max(np.abs(s_gpu[hit] - s_ref[hit]) / s_ref[hit]) < TOL_BF16
    kept, _, _ = abi.razor_select(ss, cc, keep)
    return kept_set_swaps(kept.cpu().numpy(), razor.scores(s_ref, c_ref), keep, band=4 * TOL_BF16)


def test_tiny_refill_pass_and_selection():
    """Tiny layer: the Refill pass's layer output, and its statistics and
    kept set on the decided tokens (selection and promoted expert decided by
    a logit margin above 1e-3), always compared with the oracle."""
    wl = synth.WORKLOADS["tiny"]
    w = {n: t.to(DEV) for n, t in synth.make_weights(wl, seed=0).items()}
    x = synth.make_tokens(wl, wl.T_prefill, seed=0).to(DEV)
    layer = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill, extra=1)
    ss = torch.zeros(wl.E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=DEV)
    y = layer.refill_pass(x, ss, cc)
    ref = _oracle_tokens(wl, w, x, extra=1)
    ok = ref["route"]["margin"] > 1e-3
    assert rel_err(f64(y)[ok], ref["y"][ok]) < TOL_BF16
    assert int(cc.sum()) == wl.T_prefill * wl.k
    dec = np.nonzero(ref["route"]["set_margin"] > 1e-3)[0]
    assert len(dec) >= wl.T_prefill // 2
    _check_refill_stats(layer, x, ref["route"], ref["perm"], ref["f"], wl.k, wl.E, wl.E // 2, dec)
    assert abi.moe_device_status() == 0


def test_refill_full_row_additive(bf16_layer):
    """One packed row of T=32768 tokens (the Refill workload) in the bench's
    launch configuration: statistics are additive (full pass == sum of four
    chunk passes) and every selected assignment is counted once."""
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


@pytest.mark.slow
def test_refill_full_row_vs_oracle(bf16_layer):
    """The Refill workload at full size against the float64 oracle: one row
    of T=32768 tokens, E=512, top-10 plus the promoted rank-11 expert, keep
    256.  The oracle routes all tokens and computes every permuted row's
    expert output (per-expert BLAS), then the Refill statistics in closed
    form.  (1) On the decided tokens (about 99 % of the row) the GPU pass
    gives bit-exact counts, per-expert sums of squares within 2e-2 and the
    oracle's kept set up to swaps inside the band at the 256/257 boundary.
    (2) The GPU pass over the whole row keeps the same set, up to band swaps,
    as the oracle over the whole row."""
    wl, w = bf16_layer
    wr = synth.WORKLOADS["refill"]
    T, keep = wr.T_prefill, wr.keep
    x = synth.make_tokens(wr, T, seed=0, device=DEV)
    layer = MoELayer(w, wl.k, "bf16", T_max=T, extra=1)
    xs = f64(x)
    r = moe.route(xs, f64(w["w_router"]), f64(w["bias"]), wl.k, extra=1)
    perm = moe.permute(r["idx"], wl.E)
    f, _ = moe.routed_outputs(xs, perm, expert_fn_bf16(w, wl.I, cache=False))
    del xs
    dec = np.nonzero(r["set_margin"] > 1e-3)[0]
    assert len(dec) > 0.97 * T
    _check_refill_stats(layer, x, r, perm, f, wl.k, wl.E, keep, dec)
    # the whole row, undecided tokens included
    ss = torch.zeros(wl.E, dtype=torch.float64, device=DEV)
    cc = torch.zeros(wl.E, dtype=torch.int64, device=DEV)
    layer.refill_pass(x, ss, cc)
    s_all, c_all = _refill_oracle_stats(r, perm, f, wl.k, wl.E, np.arange(T))
    n_und = T - len(dec)
    assert int(np.abs(cc.cpu().numpy() - c_all).sum()) <= 2 * n_und
    kept, _, _ = abi.razor_select(ss, cc, keep)
    kept_set_swaps(kept.cpu().numpy(), razor.scores(s_all, c_all), keep, band=4 * TOL_BF16)
    assert abi.moe_device_status() == 0
