"""AWQ W4A16 asymmetric, group 32 along the input dimension, float64 oracle.

Test infrastructure (see the package docstring).

Source: Qwen3.8-Flash-Next-AWQ-g32 card.
* "Checkpoint": 4-bit weights with 16-bit activations, asymmetric (an
  integer zero point per group), groups of 32 inputs, the AWQ GEMM packing;
  all three projections of every routed expert are quantised, with FP16
  scales.
* "Calibration": each scale is first rounded to FP16, then the code of a
  weight is its rounded quotient by the scale plus the zero point, clipped
  to 0..15.

The inverse of that code rule is w = (q - z) * s; the kernel produces it in
FP16, so the oracle's dequantised weight is fp16_rn((q - z) * s), computed
exactly in float64 and rounded once (|q - z| <= 15 has 4 significant bits and
s has 11, so the product is exact in float64).

BF16 mode ("Loading requirements", stock-runtime paragraph): a runtime that
computes in BF16 rounds the FP16 expert scales to BF16 on load (at most 0.4 %
relative per scale) and then forms the weights in BF16, so the weight is
bf16_rn((q - z) * bf16_rn(s)) (again one exact product, rounded once).

Layout (the pages name "GEMM packing" without its bit layout; this library's
reading, also stated in include/moe.h):
* A projection with input dim K and output dim N is stored input-major:
  qweight [K, N/8] int32; word w of row k holds the codes of output columns
  8w .. 8w+7, column 8w+i in bits 4i .. 4i+3.
* qzeros [K/32, N/8] int32 packed the same way; scales [K/32, N] FP16.
Interchange with real AWQ checkpoints (which may order the nibbles of a word
differently) is parity unpinned: no checkpoint is available.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, f32_to_bf16, f64_to_f16

GROUP = 32


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., N] codes 0..15 -> [..., N/8] int32, column 8w+i in bits 4i..4i+3."""
    c = np.asarray(codes, np.int64)
    assert c.shape[-1] % 8 == 0
    if np.any((c < 0) | (c > 15)):
        raise ValueError("codes must be in [0, 15]")
    c = c.reshape(*c.shape[:-1], c.shape[-1] // 8, 8)
    word = np.zeros(c.shape[:-1], np.int64)
    for i in range(8):
        word |= c[..., i] << (4 * i)
    return word.astype(np.uint32).view(np.int32)


def unpack_nibbles(words: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles: [..., N/8] int32 -> [..., N] codes (int64)."""
    w = np.asarray(words, np.int32).view(np.uint32).astype(np.int64)
    out = np.empty((*w.shape, 8), np.int64)
    for i in range(8):
        out[..., i] = (w >> (4 * i)) & 0xF
    return out.reshape(*w.shape[:-1], w.shape[-1] * 8)


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round values that are exact in binary32 to BF16 (nearest, ties to
    even), returned as float64."""
    return bf16_to_f64(f32_to_bf16(np.asarray(v, np.float64).astype(np.float32)))


def dequant(qweight: np.ndarray, qzeros: np.ndarray, scales: np.ndarray, mode: str = "fp16") -> np.ndarray:
    """W[k, n] = fp16_rn((q[k,n] - z[k//32, n]) * s[k//32, n]) (mode "fp16"),
    or bf16_rn((q - z) * bf16_rn(s)) (mode "bf16"), returned as float64
    [K, N] (input-major, as stored)."""
    q = unpack_nibbles(qweight)
    z = unpack_nibbles(qzeros)
    s = np.asarray(scales, np.float16).astype(np.float64)
    K, N = q.shape
    g = np.arange(K) // GROUP
    if mode == "bf16":
        # both products are exact in binary32: 4 x 8 significant bits
        return bf16_round((q - z[g]).astype(np.float64) * bf16_round(s)[g])
    if mode != "fp16":
        raise ValueError(mode)
    exact = (q - z[g]).astype(np.float64) * s[g]
    return f64_to_f16(exact).astype(np.float64)


def quantize(w: np.ndarray, scales: np.ndarray, zeros: np.ndarray) -> np.ndarray:
    """Code rule of the card: q = clip(round(w / s + z), 0, 15), with s already
    FP16 and round = round half to even.  w [K, N] float64, scales [K/32, N]
    FP16, zeros [K/32, N] int -> codes [K, N] int64."""
    w = np.asarray(w, np.float64)
    K, _ = w.shape
    g = np.arange(K) // GROUP
    s = np.asarray(scales, np.float16).astype(np.float64)[g]
    z = np.asarray(zeros, np.int64)[g]
    return np.clip(np.rint(w / s + z), 0, 15).astype(np.int64)


def expert_weights_out_in(qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, e: int, I: int, mode: str = "fp16"):
    """Dequantised float64 (w_gate [I,H], w_up [I,H], w_down [H,I]) of expert e,
    in the out x in orientation the MoE oracle uses.  The stored gate/up
    projection has N = 2I output columns: gate columns 0..I-1, up I..2I-1."""
    wgu = dequant(qw_gu[e], qz_gu[e], sc_gu[e], mode)  # [H, 2I]
    wd = dequant(qw_d[e], qz_d[e], sc_d[e], mode)  # [I, H]
    return wgu[:, :I].T, wgu[:, I:].T, wd.T
