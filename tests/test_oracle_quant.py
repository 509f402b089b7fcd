"""Pins for oracle/awq.py and oracle/nvfp4.py: round trips, exact special
cases, error bounds of the rounding rules, and torch conversions."""

import numpy as np
import pytest
import torch

from oracle import awq, formats, nvfp4


def test_awq_pack_layout_and_round_trip():
    codes = np.arange(1, 9).reshape(1, 8)
    w = awq.pack_nibbles(codes)
    assert w.view(np.uint32)[0, 0] == 0x87654321
    rng = np.random.default_rng(0)
    c = rng.integers(0, 16, (64, 96))
    assert np.array_equal(awq.unpack_nibbles(awq.pack_nibbles(c)), c)
    words = rng.integers(-2 ** 31, 2 ** 31, (7, 5), dtype=np.int64).astype(np.int32)
    assert np.array_equal(awq.pack_nibbles(awq.unpack_nibbles(words)), words)


def _awq_case(rng, K=64, N=32, lo_scale=0.0):
    q = rng.integers(0, 16, (K, N))
    z = rng.integers(0, 16, (K // 32, N))
    s = np.abs(rng.standard_normal((K // 32, N)) * 0.02).astype(np.float16)
    if lo_scale:
        s = np.maximum(s, np.float16(lo_scale))
    return q, z, s


def test_awq_dequant_zero_at_zero_point_and_vs_torch_half():
    rng = np.random.default_rng(1)
    q, z, s = _awq_case(rng)
    W = awq.dequant(awq.pack_nibbles(q), awq.pack_nibbles(z), s)
    g = np.arange(q.shape[0]) // 32
    # (q - z) * s with q = z is exactly zero
    qz = z[g]
    assert np.all(awq.dequant(awq.pack_nibbles(qz), awq.pack_nibbles(z), s) == 0)
    # exact product in float32, rounded once to half by torch
    prod = torch.from_numpy((q - z[g]).astype(np.float32) * s[g].astype(np.float32))
    assert np.array_equal(W, prod.to(torch.float16).double().numpy())


def test_awq_dequant_bf16_mode_vs_torch_bfloat16():
    """BF16 mode: the scale rounded to BF16 once, then one BF16 product --
    torch's own bfloat16 conversion and multiplication on the CPU give the
    same bits; q = z gives 0; a unit code difference gives the rounded scale,
    whose change is within the card's 0.4 % per scale."""
    rng = np.random.default_rng(3)
    q, z, s = _awq_case(rng, K=96, N=40)
    W = awq.dequant(awq.pack_nibbles(q), awq.pack_nibbles(z), s, mode="bf16")
    g = np.arange(q.shape[0]) // 32
    s_bf = torch.from_numpy(s[g].astype(np.float32)).to(torch.bfloat16)
    d_bf = torch.from_numpy((q - z[g]).astype(np.float32)).to(torch.bfloat16)  # |q - z| <= 15: exact
    assert np.array_equal(W, (d_bf * s_bf).double().numpy())
    assert np.all(awq.dequant(awq.pack_nibbles(z[g]), awq.pack_nibbles(z), s, mode="bf16") == 0)
    one = np.minimum(z[g] + 1, 15)
    unit = awq.dequant(awq.pack_nibbles(one), awq.pack_nibbles(z), s, mode="bf16")
    m = one - z[g] == 1
    s64 = s[g].astype(np.float64)
    assert np.array_equal(unit[m], s_bf.double().numpy()[m])
    nz = m & (s64 > 0)
    assert np.max(np.abs(unit[nz] - s64[nz]) / s64[nz]) <= 0.004
    # the two modes differ (BF16 keeps 8 significant bits, FP16 11)
    assert not np.array_equal(W, awq.dequant(awq.pack_nibbles(q), awq.pack_nibbles(z), s))


def test_awq_quantize_inverts_dequant_and_error_bound():
    rng = np.random.default_rng(2)
    q, z, s = _awq_case(rng, K=128, N=64, lo_scale=2.0 ** -10)
    W = awq.dequant(awq.pack_nibbles(q), awq.pack_nibbles(z), s)
    assert np.array_equal(awq.quantize(W, s, z), q)
    # in-range weights come back within half a step
    g = np.arange(128) // 32
    lo = (0 - z[g]) * s[g].astype(np.float64)
    hi = (15 - z[g]) * s[g].astype(np.float64)
    w = lo + rng.uniform(0, 1, lo.shape) * (hi - lo)
    qq = awq.quantize(w, s, z)
    back = (qq - z[g]) * s[g].astype(np.float64)
    assert np.all(np.abs(back - w) <= 0.5 * s[g].astype(np.float64) * (1 + 1e-12))
    # clipping outside the code range
    assert np.all(awq.quantize(lo - 10 * s[g].astype(np.float64), s, z) == 0)
    assert np.all(awq.quantize(hi + 10 * s[g].astype(np.float64), s, z) == 15)


def test_nvfp4_pack_layout():
    c = np.array([[1, 2, 3, 4]], np.uint8)
    assert list(nvfp4.pack(c)[0]) == [0x21, 0x43]
    rng = np.random.default_rng(3)
    cc = rng.integers(0, 16, (5, 32)).astype(np.uint8)
    assert np.array_equal(nvfp4.unpack(nvfp4.pack(cc)), cc)


def test_nvfp4_zero_tensor_and_zero_block():
    c, sb, g = nvfp4.quantize(np.zeros((3, 32), np.float32))
    assert g == 0 and np.all(c == 0) and np.all(sb == 0)
    v = np.random.default_rng(4).standard_normal((2, 48)).astype(np.float32)
    v[1, 16:32] = 0
    c, sb, g = nvfp4.quantize(v)
    assert np.all(c[1, 16:32] == 0) and sb[1, 1] == 0


def test_nvfp4_grid_values_round_trip_exactly():
    # s_g a power of two, block scales E4M3 values, elements on the E2M1
    # grid, each block holding a +-6 element: every division is exact
    rng = np.random.default_rng(5)
    rows, K = 8, 64
    s_g = np.float32(2.0 ** -12)
    sb_codes = rng.integers(0x20, 0x7F, (rows, K // 16)).astype(np.uint8)
    sb_codes[0, 0] = 0x7E  # one block at 448, so amax = 6 * 448 * s_g
    ecodes = rng.integers(0, 16, (rows, K)).astype(np.uint8)
    ecodes[:, ::16] = 0x7  # +6 in every block
    v = nvfp4.dequant(ecodes, sb_codes, s_g).astype(np.float32)
    c, sb, g = nvfp4.quantize(v)
    assert g == s_g
    assert np.array_equal(sb, sb_codes)
    # -0 and +0 decode equal; compare values
    assert np.array_equal(formats.e2m1_to_f64(c), formats.e2m1_to_f64(ecodes))


def test_nvfp4_error_bound_and_block_max():
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)))).astype(np.float32)
    c, sb, g = nvfp4.quantize(v)
    back = nvfp4.dequant(c, sb, g)
    scale = np.repeat(formats.e4m3_to_f64(sb), 16, axis=1) * np.float64(g)
    # the largest E2M1 gap is 2 (between 4 and 6): error <= 1 step-scale
    assert np.all(np.abs(back - v) <= 1.0 * scale * (1 + 1e-6))
    # the tensor's largest element lands on code +-6 at block scale 448
    i = np.unravel_index(np.argmax(np.abs(v)), v.shape)
    assert sb[i[0], i[1] // 16] == 0x7E
    assert (c[i] & 0x7) == 0x7


def test_nvfp4_static_scale_saturates():
    v = np.array([[100.0] + [0.0] * 15], np.float32)
    c, sb, g = nvfp4.quantize(v, s_g=np.float32(1e-3))  # 6*448*1e-3 = 2.688 < 100
    assert sb[0, 0] == 0x7E and c[0, 0] == 0x7


def test_w4a4_experts_compose_pinned_pieces():
    """The W4A4 expert path equals the pinned SwiGLU expert run on the
    globally fake-quantised activations, with h fake-quantised as ONE tensor
    over all permuted rows (not per expert) before the down projection."""
    from oracle import moe
    rng = np.random.default_rng(7)
    T, H, I, E, k = 24, 64, 32, 3, 2
    x = rng.standard_normal((T, H)).astype(np.float32).astype(np.float64)
    wgu = rng.standard_normal((E, 2 * I, H)) / 8
    wd = rng.standard_normal((E, H, I)) / 6
    deq, _ = nvfp4.quantize_expert_weights(wgu, wd)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    perm = moe.permute(idx, E)
    f, h, (s_x, s_h) = nvfp4.routed_outputs_w4a4(x, perm, deq)
    xq = nvfp4.fake_quant(x.astype(np.float32))
    h_ref = np.zeros_like(h)
    for e in range(E):
        a, b = perm["offsets"][e], perm["offsets"][e + 1]
        _, h_ref[a:b] = moe.swiglu_expert(xq[perm["row_token"][a:b]], *deq(e))
    assert np.allclose(h, h_ref, rtol=1e-12, atol=1e-12)
    # h is rounded to BF16 (torch's rounding) before it is quantised, as one tensor
    h16 = torch.from_numpy(h.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert s_h == nvfp4.global_scale(h16)  # one scale for all rows
    hq = nvfp4.fake_quant(h16)
    for e in range(E):
        a, b = perm["offsets"][e], perm["offsets"][e + 1]
        assert np.allclose(f[a:b], hq[a:b] @ deq(e)[2].T, rtol=1e-12, atol=1e-12)
    # a static activation scale is used as given (a power-of-two factor would be
    # absorbed exactly by the block scales; a 20x smaller one saturates them)
    f2, _, (sx2, sh2) = nvfp4.routed_outputs_w4a4(x, perm, deq, act_gs=(s_x / 20, s_h / 20))
    assert sx2 == np.float32(s_x / 20) and not np.allclose(f2, f)


def test_w4a4_group_products_are_exact_integers():
    """The identity the NVFP4 decode GEMVs rest on: inside one 16-element
    group both operands are E2M1 values times one scale, 2*e2m1 is an integer
    in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}, so sum (2w)(2x) is an exact
    integer of at most 16*144 in magnitude, and the dot product of the
    dequantised operands equals sum_groups int * s_bw * s_bx * s_gw * s_gx / 4
    exactly (float64)."""
    rng = np.random.default_rng(11)
    K = 256
    w = (rng.standard_normal((3, K)) * 0.05).astype(np.float32)
    x = rng.standard_normal((1, K)).astype(np.float32)
    cw, sbw, gw = nvfp4.quantize(w)
    cx, sbx, gx = nvfp4.quantize(x)
    two_w = (2 * formats.e2m1_to_f64(cw)).astype(np.int64)
    two_x = (2 * formats.e2m1_to_f64(cx)).astype(np.int64)
    assert set(np.unique(np.abs(two_w))) <= {0, 1, 2, 3, 4, 6, 8, 12}
    deq = nvfp4.dequant(cw, sbw, gw) @ nvfp4.dequant(cx, sbx, gx)[0]
    for r in range(3):
        acc = 0.0
        for g in range(K // 16):
            isum = int(np.dot(two_w[r, 16 * g:16 * g + 16], two_x[0, 16 * g:16 * g + 16]))
            assert abs(isum) <= 16 * 144
            acc += isum * formats.e4m3_to_f64(sbw[r, g]) * formats.e4m3_to_f64(sbx[0, g])
        assert acc * float(gw) * float(gx) / 4 == pytest.approx(deq[r], rel=1e-15, abs=1e-300)


def test_bf16_integer_bit_patterns_used_by_the_awq_bf16_mode():
    """0x4300 | q is the BF16 value 128 + q for every code q in 0..15, and the
    difference of two such values is q - z exactly (integers below 256 are
    exact in BF16), so one rounding remains: the product with the scale."""
    q = np.arange(16, dtype=np.uint16)
    vals = formats.bf16_to_f64(np.uint16(0x4300) | q)
    assert np.array_equal(vals, 128.0 + q)
    d = vals[:, None] - vals[None, :]
    assert np.array_equal(formats.bf16_to_f64(formats.f32_to_bf16(d.astype(np.float32))), d)
    # the FP16 pattern of the FP16 mode: 0x6400 | q is 1024 + q
    assert np.array_equal(formats.f16_to_f64((np.uint16(0x6400) | q).view(np.float16)), 1024.0 + q)


def _hand_bank(E, H, I):
    """Hand-built integer expert weights, out x in: gate [E, I, H], up
    [E, I, H], down [E, H, I], every entry in -8..7 and the three
    projections different from one another (and not symmetric), so that a
    swapped half, a missing transpose or a wrong expert index changes the
    result."""
    i = np.arange(I)[:, None]
    h = np.arange(H)[None, :]
    e = np.arange(E)[:, None, None]
    gate = ((3 * i + h + 5 * e) % 16) - 8
    up = 7 - ((i + 5 * h + 3 * e) % 16)
    down = ((7 * h.T + 3 * i.T + e) % 16) - 8  # [E, H, I]
    return gate.astype(np.int64), up.astype(np.int64), down.astype(np.int64)


def test_awq_expert_bank_split_and_orientation():
    """expert_weights_out_in against the library's documented AWQ layout,
    built by hand: the stored gate/up projection is input-major [H, 2I] with
    output columns 0..I-1 the gate and I..2I-1 the up projection; down is
    stored [I, H].  Zero points 8 and power-of-two scales (1 for gate/up
    groups, 1/2 for down) make every dequantised weight an exact small
    number, so the oracle must return exactly the hand-built matrices."""
    E, H, I = 3, 64, 32
    gate, up, down = _hand_bank(E, H, I)
    codes_gu = np.concatenate([gate, up], axis=1).transpose(0, 2, 1) + 8  # [E, H, 2I] input-major
    codes_d = down.transpose(0, 2, 1) + 8  # [E, I, H]
    qw_gu = np.stack([awq.pack_nibbles(c) for c in codes_gu])
    qw_d = np.stack([awq.pack_nibbles(c) for c in codes_d])
    qz_gu = np.stack([awq.pack_nibbles(np.full((H // 32, 2 * I), 8)) for _ in range(E)])
    qz_d = np.stack([awq.pack_nibbles(np.full((I // 32, H), 8)) for _ in range(E)])
    sc_gu = np.ones((E, H // 32, 2 * I), np.float16)
    sc_d = np.full((E, I // 32, H), 0.5, np.float16)
    for e in range(E):
        wg, wu, wd = awq.expert_weights_out_in(qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, e, I)
        assert wg.shape == (I, H) and wu.shape == (I, H) and wd.shape == (H, I)
        assert np.array_equal(wg, gate[e])
        assert np.array_equal(wu, up[e])
        assert np.array_equal(wd, 0.5 * down[e])


def test_nvfp4_expert_weights_one_global_scale_per_projection():
    """quantize_expert_weights: gate, up and down of every expert are three
    tensors, each with the global scale amax / (6 * 448) of its own values
    (one FP32 scale per tensor), and the dequantised gate / up / down come
    back in out x in orientation close to their own source rows."""
    rng = np.random.default_rng(11)
    E, H, I = 2, 64, 32
    amax = {}
    gu = np.empty((E, 2 * I, H))
    wd = np.empty((E, H, I))
    for e in range(E):
        # each tensor's largest magnitude sits at a known place, with a known value
        for name, shape, peak in (("gate", (I, H), 0.5 * (e + 1)), ("up", (I, H), 3.0 * (e + 1)),
                                  ("down", (H, I), 0.125 * (e + 2))):
            m = rng.uniform(-0.9, 0.9, shape) * peak
            m[1, 2] = -peak
            amax[(e, name)] = peak
            if name == "gate":
                gu[e, :I] = m
            elif name == "up":
                gu[e, I:] = m
            else:
                wd[e] = m
    gu = gu.astype(np.float32).astype(np.float64)
    wd = wd.astype(np.float32).astype(np.float64)
    deq, raw = nvfp4.quantize_expert_weights(gu, wd)
    for e in range(E):
        scales = []
        for name in ("gate", "up", "down"):
            s_g = raw[(e, name)][2]
            assert s_g == np.float32(np.float32(amax[(e, name)]) / np.float32(2688.0)), (e, name)
            scales.append(s_g)
        assert len(set(scales)) == 3
        wg, wu, wdd = deq(e)
        assert wg.shape == (I, H) and wu.shape == (I, H) and wdd.shape == (H, I)
        for got, src, name in ((wg, gu[e, :I], "gate"), (wu, gu[e, I:], "up"), (wdd, wd[e], "down")):
            # a 16-element group keeps its largest value within one E2M1 step and
            # the E4M3 scale rounding: far below the gap between the tensors' ranges
            assert np.max(np.abs(got - src)) <= 0.25 * amax[(e, name)], name
