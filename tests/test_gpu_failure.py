"""Failure handling on the device without a fault: a bounded wait that
nothing completes runs out, records MOE_ERR_TIMEOUT in the device status
word, stops the other roles of its CTA through the abort flag, drains its
in-flight copy and the tensor core, frees its tensor memory and returns;
the context then still runs a parity case."""

import time

import numpy as np
import pytest
import torch

from bit_expert_gemm_b200 import MoELayer, abi, synth
from oracle import moe
from tests.helpers import expert_fn_bf16, f64, rel_err, shared_fn

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tiny_layer_parity():
    wl = synth.WORKLOADS["tiny"]
    w = {n: t.to(DEV) for n, t in synth.make_weights(wl, seed=0).items()}
    x = synth.make_tokens(wl, wl.T_prefill, seed=0).to(DEV)
    y = MoELayer(w, wl.k, "bf16", T_max=wl.T_prefill).forward(x)
    ref = moe.moe_layer(f64(x), f64(w["w_router"]), f64(w["bias"]), wl.k, expert_fn_bf16(w, wl.I), shared_fn(w))
    ok = ref["route"]["margin"] > 1e-3
    return rel_err(f64(y)[ok], ref["y"][ok])


@pytest.mark.parametrize("limit_us", [2000, 20000])
def test_bounded_wait_times_out_and_context_survives(limit_us):
    torch.cuda.synchronize()
    assert abi.moe_device_status(clear=True) == abi.MOE_OK
    t0 = time.perf_counter()
    res = abi.moe_selftest_bounded_wait(limit_us)
    status = abi.moe_device_status(clear=True)  # synchronises
    dt = time.perf_counter() - t0
    assert status == abi.MOE_ERR_TIMEOUT
    assert res.cpu().tolist() == [1, 1]  # the waiting role gave up, the other stopped on the abort flag
    assert dt >= limit_us * 1e-6  # not before the limit
    assert dt < 100 * limit_us * 1e-6 + 1.0  # the second role did not sit out its own 100x longer limit
    assert abi.moe_device_status(clear=False) == abi.MOE_OK  # cleared
    # the context is intact: a parity case runs and matches the oracle
    assert _tiny_layer_parity() <= 2e-2
    assert abi.moe_device_status(clear=False) == abi.MOE_OK
