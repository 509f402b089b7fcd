"""Number formats of the expert weights, scales and activations.

Test infrastructure (see the package docstring).  Every converter here is
written from the bit-field definition of its format; the tests pin each one
against an independent library conversion (torch) and against hand-picked
values from the format definitions.

Formats and where the pages name them
-------------------------------------
* BF16 -- expert, router and shared-expert weights of the base and RAZOR
  checkpoints (RAZOR-65B model card, property table "Weight dtype").
* FP16 -- AWQ expert scales and the non-routed tensors stored in FP16
  (router and shared expert) of the AWQ g32 card, section "Checkpoint" and
  its paragraph on those tensors; activations of that card's FP16 compute.
* FP8 E4M3 (the finite-only "FN" variant, max 448) -- NVFP4 block scales
  (NVFP4 card, component table: one FP8 scale per group of 16).
* FP4 E2M1 -- NVFP4 element codes (same table: 4-bit weights and activations).
"""

from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# BF16: the upper 16 bits of an IEEE binary32.
# ----------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact BF16 -> float64 (bits: uint16 array).  A BF16 value is the
    binary32 whose low 16 bits are zero, so widening is exact."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # NaN patterns widen to NaN
        return u32.view(np.float32).astype(np.float64)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """binary32 -> BF16 bits, round to nearest, ties to even; NaN stays NaN."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    rounded = np.where(nan, np.uint16(0x7FC0), rounded)
    return rounded.astype(np.uint16)


def f64_to_bf16_values(x: np.ndarray) -> np.ndarray:
    """float64 -> the nearest BF16 value (ties to even), as float64, rounded
    once from the float64 value (not through binary32).  For finite values
    whose magnitude is inside BF16's normal range, which is all that the
    oracle rounds: with x = m * 2^e, 0.5 <= |m| < 1, BF16 keeps 8
    significant bits, so the result is rint(m * 256) / 256 * 2^e."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


# ----------------------------------------------------------------------------
# FP16 (IEEE binary16).  numpy's float16 is IEEE binary16 with correctly
# rounded conversions; the tests pin it against torch.float16.
# ----------------------------------------------------------------------------


def f16_to_f64(bits_or_vals: np.ndarray) -> np.ndarray:
    a = np.asarray(bits_or_vals)
    if a.dtype == np.uint16:
        a = a.view(np.float16)
    return a.astype(np.float64)


def f64_to_f16(x: np.ndarray) -> np.ndarray:
    """float64 -> binary16, round to nearest even (single rounding)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


# ----------------------------------------------------------------------------
# FP8 E4M3, finite-only variant: 1 sign, 4 exponent (bias 7), 3 mantissa bits.
# Exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN; no
# infinities; largest finite magnitude 1.75 * 2^8 = 448.
# ----------------------------------------------------------------------------


def _e4m3_table() -> np.ndarray:
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = s * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_VALUES = _e4m3_table()
E4M3_MAX = 448.0


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def _encode_nearest_even(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid point nearest to each mag (grid ascending, indices are
    codes); a tie goes to the even code.  mag above the last grid point maps
    to the last point (saturation)."""
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")  # first grid >= mag
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_hi = np.abs(grid[hi] - mag)
    d_lo = np.abs(mag - grid[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    return np.where(pick_lo, lo, hi)


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    """binary32 -> E4M3 code, round to nearest even, saturating to +-448
    (the 'satfinite' behaviour: out-of-range finite values clamp to the
    largest finite code instead of becoming NaN)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    grid = E4M3_VALUES[:0x7F]  # codes 0 .. 0x7E, ascending, 0 .. 448
    mag = np.minimum(np.abs(x), E4M3_MAX)
    code = _encode_nearest_even(mag, grid).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << np.uint8(7)
    return (code | sign).astype(np.uint8)


# ----------------------------------------------------------------------------
# FP4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit.  Magnitudes of codes
# 0..7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
# ----------------------------------------------------------------------------


def _e2m1_table() -> np.ndarray:
    vals = np.empty(16, dtype=np.float64)
    for code in range(16):
        s = -1.0 if code & 0x8 else 1.0
        e = (code >> 1) & 0x3
        m = code & 0x1
        vals[code] = s * (m * 0.5 if e == 0 else (1.0 + m * 0.5) * 2.0 ** (e - 1))
    return vals


E2M1_VALUES = _e2m1_table()
E2M1_MAX = 6.0


def e2m1_to_f64(codes: np.ndarray) -> np.ndarray:
    return E2M1_VALUES[np.asarray(codes, dtype=np.uint8) & 0xF]


def f32_to_e2m1(x: np.ndarray) -> np.ndarray:
    """binary32 -> E2M1 code (uint8 holding one nibble), round to nearest even,
    saturating to +-6.  The sign bit follows the sign of the input, so a
    negative value that rounds to zero gives the negative-zero code 0x8."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    grid = E2M1_VALUES[:8]
    mag = np.minimum(np.abs(x), E2M1_MAX)
    code = _encode_nearest_even(mag, grid).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << np.uint8(3)
    return (code | sign).astype(np.uint8)
