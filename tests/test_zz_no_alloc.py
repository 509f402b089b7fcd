"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (they receive only input and output buffers from their host
framework), with its scratch in a fixed array inside the library.

Checked against moe_permute (which takes a caller workspace) on two calls in
a row with different routings, so that a second call reading stale scratch
from the first would show; the outputs are integers and must match bit for
bit.  This file is collected last so that a run stopping at its first
failure has already run every other test."""

import pytest
import torch

from bit_expert_gemm_b200 import abi, synth


@pytest.mark.gpu
def test_permute_noalloc_matches_permute_on_two_calls_in_a_row():
    for call, (T, E, ks) in enumerate([(4099, 512, 10), (1000, 512, 11)]):
        idx = synth.make_routing(T, E, ks, seed=100 + call).to("cuda")
        want = abi.moe_permute(idx, E)
        got = abi.moe_permute_noalloc(idx, E)
        torch.cuda.synchronize()
        for w, g in zip(want, got):
            assert torch.equal(w, g)
    assert abi.moe_device_status() == 0


def test_permute_noalloc_rejects_batches_beyond_its_scratch():
    lib = abi.load()
    # 1024 experts x ceil(32768/32) mask words = 2^20 > the 2^19-word limit; checked before any GPU work
    rc = lib.moe_permute_noalloc(None, 32768, 10, 1024, None, None, None, None)
    assert rc == abi.MOE_ERR_UNSUPPORTED
    assert "scratch limit" in lib.moe_last_error().decode()
