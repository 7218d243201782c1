"""NVFP4 codecs, quantize and dequantize -- CPU oracle (test infrastructure only).

Source passages
  * miniTE pages (news.hamidun.com, Arabic and Russian editions, "key facts"
    list): the learner runs native NVFP4 W4A4 -- 4-bit weights and
    activations.  The pages do not print the format itself.
  * www.aib.vote "miniTE report, NVFP4 RL stability", paragraph 4: the
    token-wise NVFP4 path of Transformer Engine, amax reuse.
  * The NVFP4 format definition the pages rely on: E2M1 elements, one
    unsigned E4M3 (UE4M3) scale per 16 consecutive elements along K, and one
    FP32 global scale.

Readings taken where the pages are silent:
  R1  E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}; bit 3 is the sign.
  R2  UE4M3 = E4M3 with the sign bit 0: bias 7, 3 mantissa bits, subnormals
      m * 2^-9, largest finite 448; code 0x7F (NaN) is never produced.
  R3  Packing: element 2i goes to the low nibble of byte i, 2i+1 to the high.
  R4  Global scale: S_enc = 2688 / amax (2688 = 6 * 448) in binary32, 1 when
      amax == 0, clamped to FLT_MAX if the division overflows; the stored
      decode scale is S_dec = 1 / S_enc in binary32.
  R5  Block scale: sf = UE4M3_rne_satfinite( (bamax / 6) * S_enc ), two
      binary32 operations in that order.
  R6  Element code: r = S_enc / sf (0 when sf == 0), y = x * r, code =
      E2M1_rne_satfinite(y); ties go to the even code, |y| > 6 saturates to 6,
      a negative y that rounds to zero keeps its sign (code 0x8), and a block
      whose sf is 0 is all +0 codes.
  R7  Per-token mode computes amax per row instead of per tensor, so a
      token's codes do not depend on the other tokens of the batch.

Rounding to a finite grid is written once (``_nearest_even``) and used for both
E2M1 and UE4M3: in both formats the code's lowest bit is the mantissa's lowest
bit, so "ties to even mantissa" is "ties to the even code index".
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
FLT_MAX = F32(np.finfo(np.float32).max)

# R1: E2M1 magnitudes, indexed by the 3-bit magnitude code.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0


def _e4m3_value(code: int) -> float:
    """Value of a non-negative E4M3 code (R2), from the bit fields."""
    e, m = code >> 3, code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


# R2: codes 0..126 in increasing order of value (127 = NaN is excluded).
UE4M3_VALUES = np.array([_e4m3_value(c) for c in range(127)], dtype=np.float64)
UE4M3_MAX = 448.0
assert UE4M3_VALUES[-1] == UE4M3_MAX


def _nearest_even(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each a >= 0, ties to the even index.

    Values at or above the last grid point saturate to it (satfinite).  The
    differences are exact in fp64 wherever a tie is possible (a lies between
    two neighbouring grid values of its own magnitude).
    """
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(grid, a, side="left")          # grid[hi-1] < a <= grid[hi]
    hi = np.clip(hi, 1, len(grid) - 1)
    lo = hi - 1
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(take_hi, hi, lo)
    idx = np.where(a >= grid[-1], len(grid) - 1, idx)
    return idx.astype(np.uint8)


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    """E2M1 round-to-nearest-even, saturating; returns 4-bit codes 0..15 (R1, R6)."""
    y = np.asarray(y, dtype=np.float32)
    mag = _nearest_even(np.abs(y).astype(np.float64), E2M1_MAGNITUDES)
    sign = np.signbit(y).astype(np.uint8) << 3
    return (mag | sign).astype(np.uint8)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes -> float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where((codes & 8) != 0, -mag, mag)


def ue4m3_encode(v: np.ndarray) -> np.ndarray:
    """UE4M3 round-to-nearest-even with saturation to 448, for v >= 0 (R2)."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("UE4M3 encodes non-negative finite values only")
    return _nearest_even(v.astype(np.float64), UE4M3_VALUES)


def ue4m3_decode(codes: np.ndarray) -> np.ndarray:
    """UE4M3 codes (0..126) -> float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    if np.any(codes > 126):
        raise ValueError("UE4M3 code out of the finite range")
    return UE4M3_VALUES[codes]


# ---------------------------------------------------------------- BF16 ----

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> exact float32 values."""
    bits = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32)


def is_bf16_exact(x: np.ndarray) -> bool:
    """True when every float32 in x is exactly representable in BF16."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return bool(np.all((b & 0xFFFF) == 0))


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp64 (or fp32) values to the nearest BF16, ties to even, directly
    from the input precision (no intermediate fp32 rounding).  Returns the
    rounded values as float32 (exact).  Overflow goes to +-inf."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    a = np.abs(v[nz])
    # BF16 keeps 8 significant bits; below 2^-126 the quantum is fixed at 2^-133.
    e = np.floor(np.log2(a))
    # guard against log2 rounding at exact powers of two
    e = np.where(2.0 ** e > a, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= a, e + 1, e)
    q = np.exp2(np.maximum(e, -126.0) - 7.0)            # quantum (ulp) at a
    r = np.rint(a / q) * q                                # rint = ties to even
    r = np.where(r > 3.3895313892515355e38, np.inf, r)    # BF16 max finite
    out[nz] = np.copysign(r, v[nz])
    out[~nz] = v[~nz]
    return out.astype(np.float32)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of BF16 numbers at |v| (the ulp of the BF16 value v)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(2.0 ** e > a, e - 1, e)
    e = np.where(a > 0, e, -126.0)
    return np.exp2(np.maximum(e, -126.0) - 7.0)


# ----------------------------------------------------------- quantize ----

def global_scales(amax: np.ndarray):
    """R4: (S_enc, S_dec) in binary32 from amax (any shape)."""
    amax = np.asarray(amax, dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        s_enc = np.where(amax > 0, F32(6.0 * 448.0) / np.where(amax > 0, amax, F32(1)), F32(1))
    s_enc = np.where(np.isinf(s_enc), FLT_MAX, s_enc).astype(np.float32)
    s_dec = (F32(1.0) / s_enc).astype(np.float32)
    return s_enc, s_dec


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., K] 4-bit codes -> [..., K/2] bytes; element 2i in the low nibble (R3)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def unpack_nibbles(q: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] 4-bit codes (inverse of pack_nibbles)."""
    q = np.asarray(q, dtype=np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = q & 0xF
    out[..., 1::2] = q >> 4
    return out


def quantize(x: np.ndarray, per_token: bool, amax_in=None):
    """NVFP4-quantize a BF16 matrix x [M][K] (given as exact float32 values).

    Steps, one binary32 operation each (R4-R7):
      amax   = max |x| over the tensor (or over each row when per_token),
               unless amax_in is given (amax reuse: a value computed once
               by an earlier pass is used as is)
      S_enc  = 2688 / amax ;  S_dec = 1 / S_enc
      bamax  = max |x| over each 16-element block along K
      sf     = UE4M3( (bamax / 6) * S_enc )
      r      = S_enc / sf            (0 when sf == 0)
      code   = E2M1( x * r )         (all +0 when sf == 0)

    Returns dict with q [M][K/2] uint8, sf [M][K/16] uint8 (row-major),
    s_dec and amax as float32 arrays of shape [1] (per tensor) or [M].
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim != 2 or x.shape[1] % 16 != 0:
        raise ValueError("x must be [M][K] with K a multiple of 16")
    M, K = x.shape
    absx = np.abs(x)
    if amax_in is not None:
        amax = np.asarray(amax_in, dtype=np.float32).reshape(-1)
    elif per_token:
        amax = absx.max(axis=1) if M else np.zeros(0, np.float32)
    else:
        amax = np.array([absx.max() if x.size else 0.0], dtype=np.float32)
    s_enc, s_dec = global_scales(amax)
    s_enc_row = s_enc.reshape(-1, 1) if per_token else s_enc.reshape(1, 1)

    blocks = x.reshape(M, K // 16, 16)
    bamax = np.abs(blocks).max(axis=2) if M else np.zeros((0, K // 16), np.float32)
    t = (bamax / F32(6.0)).astype(np.float32)
    t = (t * s_enc_row).astype(np.float32)
    sf = ue4m3_encode(t)
    sf_val = ue4m3_decode(sf).astype(np.float32)          # exact in binary32
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(sf == 0, F32(0), s_enc_row / np.where(sf == 0, F32(1), sf_val)).astype(np.float32)
    y = (blocks * r[:, :, None]).astype(np.float32)
    codes = e2m1_encode(y)
    codes = np.where((sf == 0)[:, :, None], np.uint8(0), codes).astype(np.uint8)
    return {
        "q": pack_nibbles(codes.reshape(M, K)),
        "sf": sf.astype(np.uint8),
        "s_dec": s_dec.astype(np.float32),
        "amax": amax.astype(np.float32),
    }


def dequantize(q: np.ndarray, sf: np.ndarray, s_dec: np.ndarray) -> np.ndarray:
    """x_hat = e2m1(code) * sf * S_dec in fp64 (exact: the product of a 3-bit,
    a 4-bit and a 24-bit significand fits in 53 bits).  s_dec is [1] or [M]."""
    codes = unpack_nibbles(q)
    M, K = codes.shape
    vals = e2m1_decode(codes).reshape(M, K // 16, 16)
    scale = ue4m3_decode(sf).reshape(M, K // 16, 1)
    s = np.asarray(s_dec, dtype=np.float64).reshape(-1, 1, 1)
    return (vals * scale * s).reshape(M, K)
