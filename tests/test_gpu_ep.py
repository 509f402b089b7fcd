"""Expert parallelism with the library's kernels, its ranks emulated in one
process on one GPU (ep.forward_emulated: every rank's layer and tokens on the
device, the two exchanges as copies between their buffers, in the order a
real exchange imposes; no kernel waits for another).  Prefill-sized batches
run the same GEMM kernels as MoELayer on the same rows, so every rank's
output must equal MoELayer's on its tokens bit for bit; a decode-sized batch
(MoELayer then takes the decode kernels) is compared with the oracle; the
Refill scoring pass (extra = 1) is compared with MoELayer.refill_pass."""

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, ep, synth
from oracle import moe
from tests.helpers import expert_fn_bf16, f64, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def bf16_weights():
    wl = synth.WORKLOADS["bf16"]
    return wl, synth.make_weights(wl, seed=0, device=DEV)


@pytest.mark.parametrize("world,T", [(1, 512), (2, 512), (4, 300)])
def test_expert_parallel_equals_layer(bf16_weights, world, T):
    wl, w = bf16_weights
    layers = [ep.ExpertParallelLayer(w, wl.k, r, world, T_max=T) for r in range(world)]
    xs = [synth.make_tokens(wl, T - 16 * r, seed=20 + r, device=DEV) for r in range(world)]
    ys = [y.clone() for y in ep.forward_emulated(layers, xs)]
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    ref_layer = MoELayer(w, wl.k, "bf16", T_max=T)
    for r in range(world):
        ref = ref_layer.forward(xs[r])
        assert torch.equal(ys[r], ref), r
        # the exchange moved every routed row: the ranks together received T*k rows per rank
        assert int(layers[r].send_counts.sum()) == xs[r].shape[0] * wl.k
    del layers


def test_expert_parallel_refill_equals_layer(bf16_weights):
    """Refill-RMS scoring with the experts split over two emulated ranks: each
    rank's statistics and outputs equal MoELayer.refill_pass on its tokens bit
    for bit (the same FP32 rows, permuted order and fixed-order sums), and the
    ranks' statistics added equal one pass over all their tokens."""
    wl, w = bf16_weights
    world, T = 2, 512
    layers = [ep.ExpertParallelLayer(w, wl.k, r, world, T_max=T, extra=1) for r in range(world)]
    xs = [synth.make_tokens(wl, T - 16 * r, seed=60 + r, device=DEV) for r in range(world)]
    stats = [(torch.zeros(wl.E, dtype=torch.float64, device=DEV), torch.zeros(wl.E, dtype=torch.int64, device=DEV))
             for _ in range(world)]
    ys = [y.clone() for y in ep.forward_emulated(layers, xs, stats=stats)]
    torch.cuda.synchronize()
    assert abi.moe_device_status() == 0
    ref_layer = MoELayer(w, wl.k, "bf16", T_max=2 * T, extra=1)
    for r in range(world):
        ss = torch.zeros_like(stats[r][0])
        cc = torch.zeros_like(stats[r][1])
        y_ref = ref_layer.refill_pass(xs[r], ss, cc).clone()
        assert torch.equal(ys[r], y_ref), r
        assert torch.equal(stats[r][1], cc), r
        assert torch.equal(stats[r][0], ss), r
        assert int(cc.sum()) == xs[r].shape[0] * wl.k
    ss = torch.zeros_like(stats[0][0])
    cc = torch.zeros_like(stats[0][1])
    ref_layer.refill_pass(torch.cat(xs), ss, cc)
    torch.cuda.synchronize()
    assert torch.equal(stats[0][1] + stats[1][1], cc)
    assert rel_err((stats[0][0] + stats[1][0]).cpu().numpy(), ss.cpu().numpy()) < 1e-9
    del layers


def test_expert_parallel_decode_batch_vs_oracle(bf16_weights):
    wl, w = bf16_weights
    world, T = 2, 16
    layers = [ep.ExpertParallelLayer(w, wl.k, r, world, T_max=T) for r in range(world)]
    xs = [synth.make_tokens(wl, T, seed=40 + r, device=DEV) for r in range(world)]
    ys = [y.clone() for y in ep.forward_emulated(layers, xs)]
    torch.cuda.synchronize()
    for r in range(world):
        ref = moe.moe_layer(f64(xs[r]), f64(w["w_router"]), f64(w["bias"]), wl.k,
                            expert_fn_bf16(w, wl.I, cache=False), shared_fn(w))
        ok = ref["route"]["margin"] > 1e-3
        assert ok.any()
        assert rel_err(f64(ys[r])[ok], ref["y"][ok]) <= 2e-2


def test_ep_plan_and_gather_rows():
    """moe_ep_plan on a hand-made permutation and moe_gather_rows, exactly."""
    E, world = 8, 4
    counts = torch.tensor([3, 0, 2, 5, 0, 0, 1, 4], dtype=torch.int32)
    off = torch.zeros(E + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(counts, 0)
    rows = int(off[-1])
    ids, sc = abi.moe_ep_plan(off.to(DEV), world, rows)
    torch.cuda.synchronize()
    experts = np.repeat(np.arange(E), counts.numpy())
    assert np.array_equal(ids.cpu().numpy(), experts % (E // world))
    assert np.array_equal(sc.cpu().numpy(), counts.numpy().reshape(world, -1).sum(1))
    src = torch.arange(7 * 16, dtype=torch.int16).view(7, 16).to(torch.bfloat16).to(DEV)
    idx = torch.tensor([6, 0, 3, 3], dtype=torch.int32, device=DEV)
    out = abi.moe_gather_rows(src, idx)
    torch.cuda.synchronize()
    assert torch.equal(out, src[idx.long()])
    assert abi.moe_device_status() == 0
