"""MX formats for the W4A8 variant: MXFP8 activations (E4M3 elements) and
MXFP4 weights (E2M1 elements), both with E8M0 block scales -- CPU oracle (test
infrastructure only).

Source passage: the miniTE pages' precision-mismatch study lists, next to the
W4A4 NVFP4 path, variants with 8-bit activations in MXFP8 (W4A8) and 16-bit
activations (W4A16) (news.hamidun.com "miniTE ... 1.39x over BF16",
mismatch findings).  They name the format only; its definition is the public
OCP Microscaling (MX) one.

Reading taken where the pages are silent:
  R17  MXFP8 activations, per the public MX definition: blocks of 32
       consecutive elements along K share one E8M0 scale X = 2^s with
       s = floor(log2(amax_block)) - 8 (8 = the exponent of E4M3's largest
       normal, 448 = 1.75 * 2^8), clamped to [-127, 127]; an all-zero block
       takes s = -127.  Each element is E4M3(V / X), round to nearest even,
       saturating at +-448 (V / X can reach 2^9 > 448); a negative value that
       rounds to zero keeps its sign (code 0x80).  E8M0 code = s + 127.
  R18  MXFP4 weights for the same variant (the block-scaled MMA that takes
       E4M3 activations takes E8M0 scales per 32 elements on both operands):
       the same rule with E2M1 elements, s = floor(log2(amax_block)) - 2
       (6 = 1.5 * 2^2), elements E2M1(V / X) round to nearest even,
       saturating at +-6.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

BLOCK = 32
E4M3_EMAX = 8


def scale_exponent(amax: np.ndarray) -> np.ndarray:
    """s = floor(log2(amax)) - 8, clamped to [-127, 127]; -127 where amax == 0.
    floor(log2) is taken exactly from the binary exponent (frexp)."""
    amax = np.asarray(amax, dtype=np.float64)
    _, p = np.frexp(amax)                    # amax = m * 2^p, m in [0.5, 1)
    s = (p - 1) - E4M3_EMAX
    s = np.where(amax > 0, s, -127)
    return np.clip(s, -127, 127).astype(np.int64)


def e4m3_encode_signed(y: np.ndarray) -> np.ndarray:
    """Signed E4M3 codes: sign << 7 | UE4M3 code of |y| (RNE, saturating)."""
    y = np.asarray(y, dtype=np.float64)
    mag = nvfp4.ue4m3_encode(np.minimum(np.abs(y), nvfp4.UE4M3_MAX)).astype(np.uint8)
    sign = (np.signbit(y)).astype(np.uint8) << 7
    return (sign | mag).astype(np.uint8)


def e4m3_decode_signed(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    mag = nvfp4.ue4m3_decode(codes & 0x7F)
    return np.where(codes & 0x80, -mag, mag)


def quantize(x: np.ndarray):
    """x [M][K] (BF16 values, K % 32 == 0) -> codes uint8 [M][K] (E4M3),
    scales uint8 [M][K/32] (E8M0)."""
    x = np.asarray(x, dtype=np.float64)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(M, K // BLOCK, BLOCK)
    s = scale_exponent(np.abs(blocks).max(axis=2))
    v = blocks / np.ldexp(1.0, s)[:, :, None]        # exact: a power-of-two scale
    codes = e4m3_encode_signed(v).reshape(M, K)
    return codes, (s + 127).astype(np.uint8)


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    M, K = codes.shape
    s = scales.astype(np.int64) - 127
    v = e4m3_decode_signed(codes).reshape(M, K // BLOCK, BLOCK)
    return (v * np.ldexp(1.0, s)[:, :, None]).reshape(M, K)


E2M1_EMAX = 2


def quantize_mxfp4(w: np.ndarray):
    """R18: w [N][K] (K % 32 == 0) -> E2M1 codes uint8 [N][K] (one per byte,
    bit 3 the sign) and E8M0 scales uint8 [N][K/32]."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = w.reshape(N, K // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=2)
    _, p = np.frexp(amax)
    s = np.clip(np.where(amax > 0, (p - 1) - E2M1_EMAX, -127), -127, 127).astype(np.int64)
    v = blocks / np.ldexp(1.0, s)[:, :, None]
    codes = nvfp4.e2m1_encode(v).reshape(N, K)
    return codes, (s + 127).astype(np.uint8)


def dequantize_mxfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    s = scales.astype(np.int64) - 127
    v = nvfp4.e2m1_decode(codes).reshape(N, K // BLOCK, BLOCK)
    return (v * np.ldexp(1.0, s)[:, :, None]).reshape(N, K)
