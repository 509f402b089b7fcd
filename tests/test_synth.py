"""The seeded synthetic inputs follow the stated recipe: reproducible for a
seed, different across seeds and batches, with the distributions the
workloads name (activations N(0, 1), weights N(0, 1/sqrt(fan_in)), router
bias N(0, 1) or N(0, 1.5), AWQ codes and zero points uniform on 0..15,
scales |N(0, 0.02)| in FP16).  CPU only; small layers of the same recipe."""

import dataclasses

import numpy as np
import torch

from bit_expert_gemm_b200 import synth


def _wl(name, **kw):
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


def test_weights_are_reproducible_and_seed_dependent():
    wl = _wl("tiny")
    a, b, c = synth.make_weights(wl, 3), synth.make_weights(wl, 3), synth.make_weights(wl, 4)
    for n in a:
        assert torch.equal(a[n], b[n]), n
        assert not torch.equal(a[n], c[n]), n
    x0 = synth.make_tokens(wl, 64, seed=1, batch=0)
    assert torch.equal(x0, synth.make_tokens(wl, 64, seed=1, batch=0))
    assert not torch.equal(x0, synth.make_tokens(wl, 64, seed=1, batch=1))
    assert not torch.equal(x0[:8], synth.make_tokens(wl, 8, seed=1, batch=0))  # T is part of the seed


def test_bf16_recipe_distributions():
    wl = _wl("bf16", E=32, H=512, I=128, I_sh=128)
    w = synth.make_weights(wl, 0)
    H, I = wl.H, wl.I
    assert w["w_router"].dtype == torch.bfloat16 and w["w_gate_up"].shape == (32, 2 * I, H)
    assert abs(w["w_gate_up"].float().std().item() * H ** 0.5 - 1) < 0.02
    assert abs(w["w_down"].float().std().item() * I ** 0.5 - 1) < 0.02
    assert abs(w["w_router"].float().std().item() * H ** 0.5 - 1) < 0.05
    assert abs(w["w_sh_down"].float().std().item() * wl.I_sh ** 0.5 - 1) < 0.05
    b = synth.make_weights(_wl("bf16", E=4096, H=64, I=64, I_sh=64), 0)["bias"]
    assert b.dtype == torch.float32 and abs(b.std().item() / 1.5 - 1) < 0.05
    x = synth.make_tokens(wl, 4096, seed=0)
    assert x.dtype == torch.bfloat16 and abs(x.float().std().item() - 1) < 0.01 and abs(x.float().mean().item()) < 0.01


def test_awq_recipe_distributions():
    wl = _wl("awq_g32", E=8, H=256, I=128, I_sh=128)
    w = synth.make_weights(wl, 0)
    assert w["w_router"].dtype == torch.float16  # FP16 activations, router and shared expert
    assert w["qw_gu"].shape == (8, 256, 2 * 128 // 8) and w["sc_gu"].shape == (8, 256 // 32, 2 * 128)
    words = w["qw_gu"].numpy().view(np.uint32).ravel()
    nib = np.stack([(words >> (4 * i)) & 0xF for i in range(8)]).ravel()
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.9 * nib.size / 16 and counts.max() < 1.1 * nib.size / 16
    zw = w["qz_d"].numpy().view(np.uint32).ravel()
    assert set(np.unique(np.stack([(zw >> (4 * i)) & 0xF for i in range(8)]))) == set(range(16))
    s = w["sc_gu"].float()
    assert bool((s >= 0).all()) and abs(s.mean().item() / (0.02 * (2 / np.pi) ** 0.5) - 1) < 0.05  # |N(0, 0.02)|
    assert synth.make_weights(_wl("awq_g32_bf16", E=2, H=64, I=64, I_sh=64), 0)["w_router"].dtype == torch.bfloat16


def test_routing_and_selection_generators():
    idx = synth.make_routing(500, 64, 10, seed=2)
    assert idx.dtype == torch.int32 and idx.shape == (500, 10)
    assert all(len(set(r.tolist())) == 10 for r in idx)  # distinct experts per token
    counts = torch.bincount(idx.flatten().long(), minlength=64)
    assert counts.max() > 4 * counts.float().median()  # skewed, Zipf-like popularity
    ss, cc = synth.make_refill_stats(512, seed=1)
    assert bool((ss[cc == 0] == 0).all()) and (cc == 0).sum() > 50
