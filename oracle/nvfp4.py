"""NVFP4 W4A4: FP4 E2M1 elements in groups of 16 along the input dimension,
one FP8 E4M3 scale per group and one FP32 global scale per tensor.

Test infrastructure (see the package docstring).

Source: Qwen3.8-Flash-Next-RAZOR-96B-A6B-NVFP4 card, component table: the
routed experts use NVFP4 for weights and activations (FP4 values in groups
of 16, an FP8 scale per group, an FP32 scale per tensor); the shared expert
and router stay BF16.  The card names the
format but not the scale recipe; this oracle takes the plainest reading that
makes every scale a decode-direction multiplier (a reading of the pages, which leave it open):

  s_g  = amax(|V|) / (6 * 448)                  float32, per tensor
  s_b  = e4m3_rn_sat(amax(|V_block|) / (6*s_g))   per 16 elements along K
  c    = e2m1_rn_sat(v / (e4m3(s_b) * s_g))      per element
  v'   = e2m1(c) * e4m3(s_b) * s_g

Every rounding decision is taken in float32 with IEEE round-to-nearest-even
operations in exactly this order (6*s_g first, then the divisions), the
precision the kernel uses, so codes compare bit for bit.  When a block's
decoded scale is zero its codes are all +0.  A caller may pass a fixed
global scale instead of the tensor's own amax (a static, calibrated scale);
block scales then saturate at 448 and codes at +-6.
"""

from __future__ import annotations

import numpy as np

from .formats import e2m1_to_f64, e4m3_to_f64, f32_to_e2m1, f32_to_e4m3

BLOCK = 16
FP4_MAX = np.float32(6.0)
FP8_MAX = np.float32(448.0)


def global_scale(v: np.ndarray) -> np.float32:
    """s_g = amax / (6 * 448) in float32."""
    amax = np.max(np.abs(np.asarray(v, np.float32))) if np.size(v) else np.float32(0)
    return np.float32(np.float32(amax) / np.float32(FP4_MAX * FP8_MAX))


def quantize(v: np.ndarray, s_g=None):
    """v [rows, K] (float32 values; K % 16 == 0) -> (codes [rows, K] uint8
    nibbles, block scale codes [rows, K/16] uint8 E4M3, s_g float32)."""
    v = np.asarray(v, np.float32)
    rows, K = v.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    if s_g is None:
        s_g = global_scale(v)
    s_g = np.float32(s_g)
    blocks = v.reshape(rows, K // BLOCK, BLOCK)
    amax_b = np.max(np.abs(blocks), axis=2)
    t = np.float32(np.float32(6.0) * s_g)
    if t > 0:
        sb_val = (amax_b / t).astype(np.float32)
    else:
        sb_val = np.zeros_like(amax_b)
    sb_code = f32_to_e4m3(sb_val)
    sb = e4m3_to_f64(sb_code).astype(np.float32)
    denom = (sb * s_g).astype(np.float32)  # [rows, K/16]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (blocks / denom[:, :, None]).astype(np.float32)
    q = np.where(denom[:, :, None] > 0, q, np.float32(0.0))
    codes = f32_to_e2m1(q).reshape(rows, K)
    return codes, sb_code, s_g


def dequant(codes: np.ndarray, sb_code: np.ndarray, s_g) -> np.ndarray:
    """v' = e2m1(c) * e4m3(s_b) * s_g, float64 [rows, K] (exact)."""
    rows, K = codes.shape
    c = e2m1_to_f64(codes).reshape(rows, K // BLOCK, BLOCK)
    sb = e4m3_to_f64(sb_code)[:, :, None]
    return (c * sb * np.float64(np.float32(s_g))).reshape(rows, K)


def pack(codes: np.ndarray) -> np.ndarray:
    """[rows, K] nibbles -> [rows, K/2] bytes, element 2j in the low nibble."""
    c = np.asarray(codes, np.uint8) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def fake_quant(v: np.ndarray, s_g=None) -> np.ndarray:
    """quantise -> dequantise, float64."""
    c, sb, g = quantize(v, s_g)
    return dequant(c, sb, g)


def routed_outputs_w4a4(x: np.ndarray, perm: dict, expert_weights_deq, act_gs=None):
    """Routed expert outputs of an NVFP4 W4A4 layer, float64.

    x [T, H] holds the 16-bit activations (as float64).  The activations are
    quantised as one tensor (global scale over all of x, or act_gs[0]); each
    expert runs SwiGLU on its rows with its dequantised weights
    (expert_weights_deq(e) -> (w_gate [I,H], w_up [I,H], w_down [H,I])); the
    intermediate h of all permuted rows is quantised as one tensor (global
    scale over all rows, or act_gs[1]) before the down projection.  h is a
    16-bit activation tensor like every other activation of the layer: it is
    rounded to BF16 before its amax and its codes are taken, so that the
    quantisation decisions are made in the same precision as the kernel's.
    Returns (f [rows, H], h [rows, I] before rounding, (s_x, s_h))."""
    from . import moe
    from .formats import bf16_to_f64, f32_to_bf16

    x32 = np.asarray(x, np.float64).astype(np.float32)
    s_x = None if act_gs is None else np.float32(act_gs[0])
    xq = fake_quant(x32, s_x)
    s_x = global_scale(x32) if act_gs is None else np.float32(act_gs[0])
    offsets, row_token = perm["offsets"], perm["row_token"]
    E = len(offsets) - 1
    R = len(row_token)
    h_all = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        wg, wu, _ = expert_weights_deq(e)
        xe = xq[row_token[a:b]]
        he = moe.silu(xe @ wg.T) * (xe @ wu.T)
        if h_all is None:
            h_all = np.zeros((R, he.shape[1]), np.float64)
        h_all[a:b] = he
    h32 = bf16_to_f64(f32_to_bf16(h_all.astype(np.float32))).astype(np.float32)
    s_h = global_scale(h32) if act_gs is None else np.float32(act_gs[1])
    hq = fake_quant(h32, s_h)
    f = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        _, _, wd = expert_weights_deq(e)
        fe = hq[a:b] @ wd.T
        if f is None:
            f = np.zeros((R, fe.shape[1]), np.float64)
        f[a:b] = fe
    return f, h_all, (s_x, s_h)


def quantize_expert_weights(w_gate_up: np.ndarray, w_down: np.ndarray):
    """Per-(expert, projection) quantisation of 16-bit weights given as
    float64 arrays w_gate_up [E, 2I, H] (gate rows then up rows) and w_down
    [E, H, I]: gate, up and down of each expert are separate tensors with
    their own global scale.  Returns a function e -> dequantised float64
    (w_gate, w_up, w_down) and the raw (codes, scale codes, global scale)
    triples as dict[(e, name)]."""
    E, I2, _ = w_gate_up.shape
    I = I2 // 2
    raw = {}
    deq = {}
    for e in range(E):
        parts = {"gate": w_gate_up[e, :I], "up": w_gate_up[e, I:], "down": w_down[e]}
        for name, wmat in parts.items():
            c, sb, g = quantize(wmat.astype(np.float32))
            raw[(e, name)] = (c, sb, g)
            deq[(e, name)] = dequant(c, sb, g)
    return (lambda e: (deq[(e, "gate")], deq[(e, "up")], deq[(e, "down")])), raw
